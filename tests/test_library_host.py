"""CPU tests of libharp's host side through the C ABI: the library loads, exports
every entry point that include/harp.h declares, and its host logic (schedule
validation, SplitMix64, signs, base mixers, theta counts) agrees with the oracle,
which was written separately.  No compute call is made without a GPU."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

from oracle import harp_oracle as O
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        src = open(os.path.join(ROOT, "include", f)).read()
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        names.update(re.findall(r"\b(harp_[a-z0-9_]+)\s*\(", src))
    return sorted(names)


def test_library_exports_every_declared_symbol():
    L = H.lib()
    names = _declared_functions()
    assert len(names) >= 13
    missing = [n for n in names if not hasattr(L, n)]
    assert not missing, missing


def test_status_strings():
    L = H.lib()
    for code, name in [(0, b"HARP_OK"), (2, b"HARP_ERR_SCHEDULE"), (4, b"HARP_ERR_NOT_MATERIALIZED"),
                       (7, b"HARP_ERR_TIMEOUT")]:
        assert L.harp_status_string(code) == name


def test_splitmix64_matches_published_and_oracle():
    got = H.splitmix64(0, 4).tolist()
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F, 0xF88BB8A8724C81EC]
    assert H.splitmix64(3003, 64).tolist() == O.splitmix64(3003, 64)


@pytest.mark.parametrize("schedule", [(8, 8), (2,) * 6, (8, 8, 8, 8), (8, 8, 8, 5, 2),
                                      (8, 8, 8, 8, 2), (8, 8, 8, 8, 7), (16, 3, 11)])
def test_theta_count_matches_oracle(schedule):
    assert H.theta_count(schedule) == O.theta_count(schedule)


@pytest.mark.parametrize("b", [2, 3, 4, 5, 7, 8, 11, 16])
def test_base_mixers_match_oracle(b):
    plan = H.Plan(b * 2, (b, 2), sign_seed=1)
    np.testing.assert_allclose(plan.base_mixer(b), O.base_mixer(b), atol=1e-14, rtol=0)


def test_qr_seed_is_honoured():
    plan = H.Plan(10, (5, 2), qr_seed=99)
    np.testing.assert_allclose(plan.base_mixer(5), O.qr_mixer(5, 99), atol=1e-14, rtol=0)


@pytest.mark.parametrize("d,schedule,seed", [(4096, (8, 8, 8, 8), 3002), (28672, (8, 8, 8, 8, 7), 1),
                                             (64, (2,) * 6, 3001)])
def test_signs_match_oracle(d, schedule, seed):
    plan = H.Plan(d, schedule, sign_seed=seed)
    np.testing.assert_array_equal(plan.signs().astype(float), O.sign_vector(d, seed))
    assert plan.shape() == (d, schedule)


@pytest.mark.parametrize("d,schedule,code", [
    (64, (8, 4), HB.HARP_ERR_SCHEDULE),            # product differs from d
    (64, (64,), HB.HARP_ERR_SCHEDULE),             # radix above 16
    (2, (1, 2), HB.HARP_ERR_SCHEDULE),             # radix below 2
    (65536, (16, 16, 16, 16), HB.HARP_ERR_INVALID_ARG),  # d above the maximum
    (1, (1,), HB.HARP_ERR_INVALID_ARG),
])
def test_plan_validation_errors(d, schedule, code):
    with pytest.raises(HB.HarpError) as e:
        H.Plan(d, schedule)
    assert e.value.status == code


def test_too_many_stages():
    with pytest.raises(HB.HarpError) as e:
        H.Plan(2 ** 17, (2,) * 17)
    assert e.value.status in (HB.HARP_ERR_SCHEDULE, HB.HARP_ERR_INVALID_ARG)


def test_int8_without_scales_rejected():
    L = H.lib()
    h = ctypes.c_void_p()
    codes = np.zeros(O.theta_count((8, 8)), dtype=np.int8)
    st = L.harp_plan_create(ctypes.byref(h), 64, HB._radices((8, 8)), 2, HB.HARP_THETA_I8,
                            codes.ctypes.data, None, 0, 0)
    assert st == HB.HARP_ERR_INVALID_ARG


def test_apply_before_materialize_is_reported_without_touching_a_device():
    L = H.lib()
    plan = H.Plan(64, (8, 8))
    st = L.harp_apply(plan.handle, ctypes.c_void_p(16), ctypes.c_void_p(16), 4, 64, 64,
                      HB.HARP_F32, HB.HARP_FORWARD, None)
    assert st == HB.HARP_ERR_NOT_MATERIALIZED
    assert b"materialize" in L.harp_last_error()
    # argument errors come first and never reach the device
    assert L.harp_apply(plan.handle, None, None, 0, 64, 64, 0, 0, None) == HB.HARP_OK
    assert L.harp_apply(plan.handle, None, None, 4, 63, 64, 0, 0, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_apply(plan.handle, None, None, 4, 64, 64, 7, 0, None) == HB.HARP_ERR_UNSUPPORTED
    assert L.harp_apply(plan.handle, None, None, 4, 64, 64, 0, 5, None) == HB.HARP_ERR_UNSUPPORTED
    assert L.harp_apply(None, None, None, 4, 64, 64, 0, 0, None) == HB.HARP_ERR_INVALID_ARG


def test_two_sided_workspace_bytes():
    assert H.workspace_bytes(28672, 8192) == 2 * 28672 * 8192 * 4
    assert H.workspace_bytes(3, 5) == 2 * 256
    assert H.workspace_bytes(0, 5) == 0


def test_destroy_null_is_ok():
    assert H.lib().harp_plan_destroy(None) == HB.HARP_OK


@pytest.mark.parametrize("schedule", [(8, 8), (8, 8, 8, 5, 2), (3, 5, 7), (2,) * 6])
def test_grad_workspace_bytes(schedule):
    # one float per block entry, each stage padded to a multiple of 4 floats (16 bytes)
    d = int(np.prod(schedule))
    plan = H.Plan(d, schedule)
    want = sum(((d // b) * b * b + 3) // 4 * 4 for b in schedule) * 4
    assert H.lib().harp_grad_workspace_bytes(plan.handle) == want
    assert H.lib().harp_grad_workspace_bytes(None) == 0


def test_grad_theta_argument_errors_before_any_device_call():
    L = H.lib()
    plan = H.Plan(64, (8, 8))
    p = ctypes.c_void_p(16)
    ws = int(L.harp_grad_workspace_bytes(plan.handle))
    args = lambda **kw: dict(dict(plan=plan.handle, x=p, g=p, rows=4, ld_x=64, ld_g=64, dtype=HB.HARP_F32,
                                  dtheta=p, ws=p, ws_bytes=ws, stream=None), **kw)

    def call(**kw):
        a = args(**kw)
        return L.harp_grad_theta(a["plan"], a["x"], a["g"], a["rows"], a["ld_x"], a["ld_g"], a["dtype"],
                                 a["dtheta"], a["ws"], a["ws_bytes"], a["stream"])

    assert call(plan=None) == HB.HARP_ERR_INVALID_ARG
    assert call(dtype=7) == HB.HARP_ERR_UNSUPPORTED
    assert call(rows=-1) == HB.HARP_ERR_INVALID_ARG
    assert call(ld_g=63) == HB.HARP_ERR_INVALID_ARG
    assert call(dtheta=None) == HB.HARP_ERR_INVALID_ARG
    assert call() == HB.HARP_ERR_NOT_MATERIALIZED


def test_apply_quant_argument_errors_before_any_device_call():
    L = H.lib()
    plan = H.Plan(4096, (8, 8, 8, 8))
    p = ctypes.c_void_p(16)

    def call(plan_h=plan.handle, x=p, rows=4, ld_x=4096, dtype=HB.HARP_BF16, q=p, ld_q=4096, s=p, ld_s=32,
             qblock=128, direction=HB.HARP_FORWARD):
        return L.harp_apply_quant(plan_h, x, rows, ld_x, dtype, q, ld_q, s, ld_s, qblock, direction, None)

    assert call(plan_h=None) == HB.HARP_ERR_INVALID_ARG
    assert call(dtype=HB.HARP_F32) == HB.HARP_ERR_UNSUPPORTED
    assert call(direction=5) == HB.HARP_ERR_UNSUPPORTED
    assert call(rows=-1) == HB.HARP_ERR_INVALID_ARG
    for qb in (16, 48, 512):
        assert call(qblock=qb) == HB.HARP_ERR_INVALID_ARG
    assert call(ld_q=4095) == HB.HARP_ERR_INVALID_ARG
    assert call(qblock=256, ld_s=15) == HB.HARP_ERR_INVALID_ARG
    assert call(rows=0, x=None, q=None, s=None) == HB.HARP_OK
    assert call(q=None) == HB.HARP_ERR_INVALID_ARG
    assert call() == HB.HARP_ERR_NOT_MATERIALIZED
    odd = H.Plan(96, (8, 4, 3))                                         # 64 does not divide 96
    assert call(plan_h=odd.handle, ld_x=96, ld_q=96, ld_s=2, qblock=64) == HB.HARP_ERR_INVALID_ARG


def test_plan_compose_argument_errors_before_any_device_call():
    L = H.lib()
    out = ctypes.c_void_p()
    keep = H.Plan(64, (8, 8))
    plans = (ctypes.c_void_p * 1)(keep.handle)
    assert L.harp_plan_compose(None, plans, 1, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_plan_compose(ctypes.byref(out), plans, 0, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_plan_compose(ctypes.byref(out), None, 1, None) == HB.HARP_ERR_INVALID_ARG
    assert not out.value


def test_wait_timeout_hook_arguments():
    L = H.lib()
    assert L.harp_test_inject_wait_timeout(0, 16) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_test_inject_wait_timeout(-1, 0) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_test_inject_wait_timeout(10, 8192) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_test_inject_wait_timeout(5, 16) == HB.HARP_OK
    assert L.harp_test_inject_wait_timeout(0, 0) == HB.HARP_OK


def test_fit_term_argument_errors_before_any_device_call():
    L = H.lib()
    p = ctypes.c_void_p(16)
    out = ctypes.c_void_p(1 << 40)
    assert L.harp_off_block_energy(p, 64, 64, HB.HARP_F32, 48, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_off_block_energy(p, 64, 63, HB.HARP_F32, 8, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_off_block_energy(p, 0, 64, HB.HARP_F32, 8, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_off_block_energy(p, 64, 64, 9, 8, out, None) == HB.HARP_ERR_UNSUPPORTED
    assert L.harp_off_block_energy(None, 64, 64, HB.HARP_F32, 8, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_off_block_energy(p, 64, 64, HB.HARP_F32, 8, ctypes.c_void_p(32), None) == HB.HARP_ERR_INVALID_ARG
    for qb in (16, 48, 512):
        assert L.harp_l_diag(p, 4, 512, 512, HB.HARP_F32, p, 512, qb, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_l_diag(p, 4, 96, 96, HB.HARP_F32, p, 96, 64, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_l_diag(p, 4, 512, 511, HB.HARP_F32, p, 512, 32, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_l_diag(p, 4, 512, 512, HB.HARP_F32, p, 511, 32, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_l_diag(p, 4, 512, 512, HB.HARP_F32, None, 512, 32, out, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_l_diag(p, 4, 512, 512, 3, p, 512, 32, out, None) == HB.HARP_ERR_UNSUPPORTED


def test_moment_check_argument_errors_before_any_device_call():
    L = H.lib()
    p = ctypes.c_void_p(16)
    out = ctypes.c_void_p(1 << 40)
    assert L.harp_moment_check(p, 4, 64, 64, 7, 0.1, 0.2, out, None, None) == HB.HARP_ERR_UNSUPPORTED
    assert L.harp_moment_check(p, -1, 64, 64, HB.HARP_F32, 0.1, 0.2, out, None, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_moment_check(p, 4, 64, 63, HB.HARP_F32, 0.1, 0.2, out, None, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_moment_check(p, 4, 64, 64, HB.HARP_F32, 0.3, 0.2, out, None, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_moment_check(p, 4, 64, 64, HB.HARP_F32, 0.1, 0.2, None, None, None) == HB.HARP_ERR_INVALID_ARG
    assert L.harp_moment_check(p, 4, 64, 64, HB.HARP_F32, 0.1, 0.2, ctypes.c_void_p(32), None, None) \
        == HB.HARP_ERR_INVALID_ARG
    assert L.harp_moment_check(None, 0, 64, 64, HB.HARP_F32, 0.1, 0.2, None, None, None) == HB.HARP_OK

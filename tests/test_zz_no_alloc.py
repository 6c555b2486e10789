"""The allocation-free two-sided entry point (harp_apply_two_sided_noalloc).

Some callers cannot allocate device memory at the moment they rotate a weight
(code inside a memory pool or arena it does not own, capture regions, host
runtimes without an allocator for plugins), so the library offers a variant of
the two-sided rotation whose workspace is a fixed array in its own device image.
These tests call it through the C ABI and hold its output to the same tolerance
as every other bf16 test: within one bf16 ordinal step of the float64 oracle's
T_U^T W T_V (tests/_parity.check_bf16), and within one step of the workspace-taking
entry point, on two calls in a row.  The file is named to be collected last.
"""
import ctypes

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB
from tests._parity import bf16_ordinal, check_bf16

pytestmark = pytest.mark.gpu


def _plan(sched, seed, sign):
    d = int(np.prod(sched))
    theta = W.draw_theta(H.theta_count(sched), 0.2236, seed)
    return H.Plan(d, sched, theta=theta, sign_seed=sign).materialize()


def _oracle_plan(sched, seed, sign):
    d = int(np.prod(sched))
    return O.make_plan(d, sched, W.draw_theta(O.theta_count(sched), 0.2236, seed), sign_seed=sign)


def _as_bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("u_sched,v_sched", [((8, 8, 7), (8, 8, 2)), ((8, 8, 8, 4), (16, 16, 8))])
def test_noalloc_matches_workspace_entry_point_twice(u_sched, v_sched):
    L = H.lib()
    pu, pv = _plan(u_sched, 41, 5), _plan(v_sched, 42, 6)
    n_out, n_in = pu.d, pv.d
    assert n_out * n_in * 8 <= L.harp_noalloc_scratch_bytes()
    rng = np.random.default_rng(n_out + n_in)
    enc = W.encode_bf16(0.02 * rng.standard_normal((n_out, n_in)))
    w = torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16).cuda()
    ref = _as_bits(H.apply_two_sided(pu, pv, w))
    wv = W.decode_bf16(enc)
    exact = O.two_sided(_oracle_plan(u_sched, 41, 5), _oracle_plan(v_sched, 42, 6), wv)
    wnorm = np.full(n_out, np.max(np.linalg.norm(wv, axis=1)))   # the two-sided tests' row-norm scale
    stream = torch.cuda.current_stream().cuda_stream
    for _ in range(2):
        out = torch.empty_like(w)
        st = L.harp_apply_two_sided_noalloc(pu.handle, pv.handle, w.data_ptr(), out.data_ptr(),
                                            n_out, n_in, n_in, HB.HARP_BF16, stream)
        assert st == HB.HARP_OK, L.harp_last_error()
        torch.cuda.synchronize()
        got = _as_bits(out)
        check_bf16(got, exact, wnorm, O.round_bf16, "noalloc against the oracle")
        assert np.abs(bf16_ordinal(got) - bf16_ordinal(ref)).max() <= 1


def test_noalloc_in_place_and_rejects_oversized_weights():
    L = H.lib()
    pu, pv = _plan((8, 8, 7), 43, 9), _plan((8, 8, 2), 44, 10)
    rng = np.random.default_rng(3)
    w = torch.from_numpy(W.encode_bf16(rng.standard_normal((448, 128))).view(np.int16)).view(torch.bfloat16).cuda()
    ref = _as_bits(H.apply_two_sided(pu, pv, w))
    stream = torch.cuda.current_stream().cuda_stream
    st = L.harp_apply_two_sided_noalloc(pu.handle, pv.handle, w.data_ptr(), w.data_ptr(), 448, 128, 128,
                                        HB.HARP_BF16, stream)
    assert st == HB.HARP_OK, L.harp_last_error()
    torch.cuda.synchronize()
    assert np.abs(bf16_ordinal(_as_bits(w)) - bf16_ordinal(ref)).max() <= 1
    big_u, big_v = _plan((16, 16, 8), 45, 11), _plan((16, 16, 9), 46, 12)   # 2048 x 2304 > limit
    x = torch.empty(2048, 2304, dtype=torch.bfloat16, device="cuda")
    st = L.harp_apply_two_sided_noalloc(big_u.handle, big_v.handle, x.data_ptr(), x.data_ptr(), 2048, 2304,
                                        2304, HB.HARP_BF16, stream)
    assert st == HB.HARP_ERR_INVALID_ARG
    assert b"static scratch" in L.harp_last_error()

"""The boundary's plan conventions on the GPU (the C ABI of include/harp.h):

* a plan is immutable once materialized: every table a kernel reads, the specialized
  d = 4096 kernel's coefficient table included, is built by harp_materialize_blocks, so the
  first calls of a freshly materialized plan may run on two streams, or from two host
  threads, with no ordering between them;
* an int8 plan (HARP technical summary §2.4: theta stored in int8) that was never
  materialized materializes on its first call, also when two first calls race.

Every result is checked against the float64 oracle (one bf16 ordinal step, tests/_parity).
"""
import threading

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from tests._parity import check_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _bits(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _rows(name, rows):
    w = W.get(name)
    enc = W.draw_encoded(w, 0, rows)
    return enc, W.decode_bf16(enc), torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16).to(DEV)


def _check(y, tr, xf, direction, what):
    check_bf16(_bits(y), tr.apply(xf, direction), np.linalg.norm(xf, axis=1), O.round_bf16, what)


def _f32_plan(name, seed_offset=0):
    w = W.get(name)
    theta = W.draw_theta(O.theta_count(w.schedule), w.theta_sigma, w.theta_seed + seed_offset)
    gp = H.Plan(w.d, w.schedule, theta=theta, sign_seed=w.sign_seed + seed_offset)
    return gp, O.Transform(O.make_plan(w.d, w.schedule, theta, sign_seed=w.sign_seed + seed_offset))


def _i8_plan(name, seed_offset=0):
    w = W.get(name)
    theta = W.draw_theta(O.theta_count(w.schedule), w.theta_sigma, w.theta_seed + seed_offset)
    codes, scales = W.quantize_theta_int8(theta, O.stage_theta_counts(w.schedule))
    gp = H.Plan(w.d, w.schedule, codes=codes, scales=scales, sign_seed=w.sign_seed + seed_offset)
    op = O.make_plan(w.d, w.schedule, codes=codes, scales=scales, sign_seed=w.sign_seed + seed_offset)
    return gp, O.Transform(op)


@pytest.mark.parametrize("seed_offset", [0, 1])
def test_first_calls_of_a_fresh_plan_on_two_streams(seed_offset):
    """C2 shape (the specialized kernel): materialize, then the plan's first two applies on
    two new streams with nothing ordering one after the other."""
    gp, tr = _f32_plan("d4096", seed_offset)
    gp.materialize()
    torch.cuda.synchronize()
    _, xf, x = _rows("d4096", 300)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    y1, y2 = torch.empty_like(x), torch.empty_like(x)
    torch.cuda.synchronize()
    with torch.cuda.stream(s1):
        gp.apply(x, y1, stream=s1)
    assert H.last_kernel() == "harp_fast_d4096_fwd_kernel"
    with torch.cuda.stream(s2):
        gp.apply(x, y2, stream=s2)
    torch.cuda.synchronize()
    _check(y1, tr, xf, "forward", "first call, stream 1")
    _check(y2, tr, xf, "forward", "first call, stream 2")
    assert np.array_equal(_bits(y1), _bits(y2))
    gp.device_status()


def test_first_calls_from_two_host_threads():
    """Two host threads, each with its own stream, start on the same freshly materialized
    plan at once (the binding releases the interpreter lock around each C call)."""
    gp, tr = _f32_plan("d4096", 2)
    gp.materialize()
    torch.cuda.synchronize()
    _, xf, x = _rows("d4096", 257)
    outs, errs = [None, None], []
    go = threading.Barrier(2)

    def run(k):
        try:
            s = torch.cuda.Stream()
            y = torch.empty_like(x)
            go.wait()
            for _ in range(3):
                gp.apply(x, y, stream=s)
            s.synchronize()
            outs[k] = y
        except Exception as e:            # surfaced below
            errs.append(e)

    th = [threading.Thread(target=run, args=(k,)) for k in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    for k in range(2):
        _check(outs[k], tr, xf, "forward", f"thread {k}")


@pytest.mark.parametrize("name,rows,direction", [("d8192_int8", 16, "forward"), ("d8192_int8", 300, "inverse"),
                                                 ("d8192_int8", 1, "inverse")])
def test_int8_plan_materializes_on_its_first_apply(name, rows, direction):
    gp, tr = _i8_plan(name)
    _, xf, x = _rows(name, rows)
    y = gp.apply(x, direction=direction)          # no materialize() before it
    torch.cuda.synchronize()
    _check(y, tr, xf, direction, f"{name} implicit materialization")
    gp.device_status()


def test_int8_first_calls_race_from_two_threads():
    gp, tr = _i8_plan("d8192_int8", 3)
    _, xf, x = _rows("d8192_int8", 40)
    outs, errs = [None, None], []
    go = threading.Barrier(2)

    def run(k):
        try:
            s = torch.cuda.Stream()
            y = torch.empty_like(x)
            go.wait()
            gp.apply(x, y, stream=s, direction="forward")
            s.synchronize()
            outs[k] = y
        except Exception as e:
            errs.append(e)

    th = [threading.Thread(target=run, args=(k,)) for k in range(2)]
    for t in th:
        t.start()
    for t in th:
        t.join()
    assert not errs, errs
    for k in range(2):
        _check(outs[k], tr, xf, "forward", f"racing first call {k}")


def test_int8_plan_materializes_on_other_entry_points():
    """harp_apply_quant, harp_apply_host and harp_apply_two_sided on fresh int8 plans."""
    gp, tr = _i8_plan("d8192_int8", 4)
    _, xf, x = _rows("d8192_int8", 24)
    q, sc = gp.apply_quant(x, 128)
    torch.cuda.synchronize()
    y = tr.forward(xf)
    deq = (q.cpu().numpy().astype(np.float64).reshape(24, -1, 128) * sc.cpu().numpy()[..., None]).reshape(24, -1)
    assert np.abs(deq - y).max() <= 0.51 * float(sc.max()) + 1e-5 * np.abs(y).max()
    gp2, tr2 = _i8_plan("d8192_int8", 5)
    enc, xf2, _ = _rows("d8192_int8", 8)
    xh = torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16)
    yh = gp2.apply_host(xh)
    check_bf16(yh.view(torch.int16).numpy().view(np.uint16), tr2.forward(xf2), np.linalg.norm(xf2, axis=1),
               O.round_bf16, "apply_host implicit materialization")
    # two-sided with both sides int8 and never materialized: U (8,8,2) on 128 rows, V (8,8,8,8,2)
    th_u = W.draw_theta(O.theta_count((8, 8, 2)), 0.2236, 77)
    cu, su = W.quantize_theta_int8(th_u, O.stage_theta_counts((8, 8, 2)))
    pu = H.Plan(128, (8, 8, 2), codes=cu, scales=su, sign_seed=78)
    opu = O.make_plan(128, (8, 8, 2), codes=cu, scales=su, sign_seed=78)
    gv, trv = _i8_plan("d8192_int8", 6)
    wt = np.random.default_rng(5).standard_normal((128, 8192)) * 0.02
    wenc = W.encode_bf16(wt)
    wv = W.decode_bf16(wenc)
    wd = torch.from_numpy(wenc.view(np.int16)).view(torch.bfloat16).to(DEV)
    out = H.apply_two_sided(pu, gv, wd)
    torch.cuda.synchronize()
    ref = O.two_sided(opu, trv.plan, wv)
    check_bf16(_bits(out), ref, np.full(128, np.max(np.linalg.norm(wv, axis=1))), O.round_bf16, "two-sided implicit")

"""GPU parity of the two-sided rotation through the column passes (harp_cols_kernel):
against the float64 oracle for fp32 and bf16 weights, bit for bit against the
transpose path (forced with HARP_KERNEL=simple; both sum every output in the same
order), ragged column counts, and the fallback when rows are not 16-byte aligned."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from tests._parity import check_bf16, check_f32
from tests.test_parity_gpu import to_dev, to_host, decode

pytestmark = pytest.mark.gpu


def _pair(schedule, seed):
    d = int(np.prod(schedule))
    theta = W.draw_theta(O.theta_count(schedule), 0.05, seed)
    gp = H.Plan(d, schedule, theta=theta, sign_seed=seed + 3)
    gp.materialize()
    return gp, O.Transform(O.make_plan(d, schedule, theta, sign_seed=seed + 3))


CASES = [((8, 8, 7), (8, 8, 2)), ((8, 8, 8, 7), (8, 2)), ((2, 8, 8), (5, 2, 8)), ((8, 5, 2, 4), (4, 4)),
         ((7, 8, 8, 8), (8, 8))]


@pytest.mark.parametrize("u_sched,v_sched", CASES)
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_two_sided_columns_vs_oracle(u_sched, v_sched, dtype):
    pu, tu = _pair(u_sched, 41)
    pv, tv = _pair(v_sched, 52)
    n_out, n_in = pu.d, pv.d
    w = np.random.default_rng(n_out + n_in).standard_normal((n_out, n_in)) * 0.02
    enc = W.encode_bf16(w) if dtype == "bf16" else w.astype(np.float32)
    out = to_host(H.apply_two_sided(pu, pv, to_dev(enc)))
    torch.cuda.synchronize()
    assert H.last_kernel() == "harp_cols_kernel"
    wf = decode(enc)
    want = tu.inverse(tv.inverse(wf).T).T
    tau = np.full(n_out, np.max(np.linalg.norm(wf, axis=1)))
    if dtype == "bf16":
        check_bf16(out, want, tau, O.round_bf16, f"two-sided {u_sched} {v_sched}")
    else:
        # the fp32 bound per row of W_out: 2e-6 of the largest row norm of W (every row
        # of the result mixes all rows of W)
        check_f32(out, want, tau, f"two-sided fp32 {u_sched} {v_sched}")


@pytest.mark.parametrize("n_in_sched", [(8, 8, 2), (5, 4, 5)])
def test_columns_match_the_transpose_path_bit_for_bit(monkeypatch, n_in_sched):
    pu, _ = _pair((8, 8, 8, 7), 61)
    pv, _ = _pair(n_in_sched, 62)
    w = np.random.default_rng(7).standard_normal((pu.d, pv.d)) * 0.02
    for enc in (W.encode_bf16(w), w.astype(np.float32)):
        monkeypatch.delenv("HARP_KERNEL", raising=False)
        a = to_host(H.apply_two_sided(pu, pv, to_dev(enc)))
        kernel = H.last_kernel()
        monkeypatch.setenv("HARP_KERNEL", "simple")
        b = to_host(H.apply_two_sided(pu, pv, to_dev(enc)))
        torch.cuda.synchronize()
        assert kernel == "harp_cols_kernel"
        np.testing.assert_array_equal(a, b)


def test_full_size_two_sided_matches_the_transpose_path_on_sampled_rows(monkeypatch):
    w4 = W.get("two_sided")
    pu, _ = _pair(w4.u_schedule, 71)
    pv, _ = _pair(w4.schedule, 72)
    wt = to_dev(W.draw_encoded(w4, 0, w4.n_out, w4.n_in))
    monkeypatch.delenv("HARP_KERNEL", raising=False)
    a = H.apply_two_sided(pu, pv, wt)
    assert H.last_kernel() == "harp_cols_kernel"
    monkeypatch.setenv("HARP_KERNEL", "simple")
    rows = torch.from_numpy(W.sample_rows(w4.n_out, 64)).to(wt.device)
    b = H.apply_two_sided(pu, pv, wt)
    torch.cuda.synchronize()
    assert torch.equal(a[rows], b[rows])
    assert torch.equal(a[-1], b[-1]) and torch.equal(a[:, -1], b[:, -1])


def test_unaligned_columns_fall_back(monkeypatch):
    monkeypatch.delenv("HARP_KERNEL", raising=False)
    pu, tu = _pair((8, 8, 7), 81)
    pv, tv = _pair((5, 2, 3), 82)             # n_in = 30: rows of fp32 not 16-byte multiples
    w = np.random.default_rng(3).standard_normal((pu.d, pv.d)) * 0.02
    enc = w.astype(np.float32)
    out = to_host(H.apply_two_sided(pu, pv, to_dev(enc)))
    torch.cuda.synchronize()
    assert H.last_kernel() != "harp_cols_kernel"
    want = tu.inverse(tv.inverse(w.astype(np.float32).astype(np.float64)).T).T
    check_f32(out, want, np.full(pu.d, np.max(np.linalg.norm(enc.astype(np.float64), axis=1))), "fallback")


@pytest.mark.parametrize("sched", [(8, 8, 8, 7), (8, 8, 2), (5, 2, 8), (2, 8, 8)])
@pytest.mark.parametrize("direction", ["forward", "inverse"])
@pytest.mark.parametrize("out", ["f32", "bf16", "in_place"])
def test_apply_columns_vs_oracle(sched, direction, out):
    gp, tr = _pair(sched, 91)
    d, ncols = gp.d, 200
    x = np.random.default_rng(d + ncols).standard_normal((d, ncols)).astype(np.float32)
    xt = to_dev(x)
    if out == "in_place":
        y = gp.apply_columns(xt, direction=direction)
    else:
        yt = torch.empty(d, ncols, device=xt.device, dtype=torch.bfloat16 if out == "bf16" else torch.float32)
        y = gp.apply_columns(xt, yt, direction=direction)
    torch.cuda.synchronize()
    assert H.last_kernel() == "harp_cols_kernel"
    want = tr.apply(x.astype(np.float64).T, direction).T          # every column
    got = to_host(y)
    cn = np.linalg.norm(x.astype(np.float64), axis=0)              # column norms
    if out == "bf16":
        check_bf16(got.T.copy(), want.T, cn, O.round_bf16, f"columns {sched} {direction}")
    else:
        check_f32(got.T, want.T, cn, f"columns {sched} {direction}")


def test_apply_ex_bf16_rows_to_f32():
    gp, tr = _pair((8, 8, 8, 8, 2), 93)
    enc = W.encode_bf16(np.random.default_rng(5).standard_normal((70, gp.d)))
    x = to_dev(enc)
    y = torch.empty(70, gp.d, device=x.device, dtype=torch.float32)
    gp.apply_ex(x, y, direction="inverse")
    torch.cuda.synchronize()
    xf = decode(enc)
    check_f32(to_host(y), tr.inverse(xf), np.linalg.norm(xf, axis=1), "apply_ex bf16 -> f32")


def test_row_sharded_two_sided_on_one_rank_equals_two_sided():
    from structured_rotations_b200.shard import two_sided_row_sharded
    pu, _ = _pair((8, 8, 8, 7), 95)
    pv, _ = _pair((8, 8, 8, 2), 96)
    w = to_dev(W.encode_bf16(np.random.default_rng(9).standard_normal((pu.d, pv.d)) * 0.02))
    a = two_sided_row_sharded(pu, pv, w)
    b = H.apply_two_sided(pu, pv, w)
    torch.cuda.synchronize()
    assert torch.equal(a, b)

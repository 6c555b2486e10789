"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle on the
same seeded inputs, for every workload, forward and inverse, at small sizes
compared in full (several tiles plus a ragged tail) and at the full sizes in the
launch configuration the bench times, compared on sampled rows plus properties
that hold at any size."""
import functools

import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB
from tests._parity import check_bf16, check_f32

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


# ------------------------------------------------------------------ helpers ---

def to_dev(enc: np.ndarray):
    if enc.dtype == np.uint16:
        return torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(enc)).to(DEV)


def to_host(t) -> np.ndarray:
    t = t.detach()
    if t.dtype == torch.bfloat16:
        return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def decode(enc: np.ndarray) -> np.ndarray:
    return W.decode_bf16(enc) if enc.dtype == np.uint16 else enc.astype(np.float64)


def theta_for(w: W.Workload, schedule=None):
    sched = schedule or w.schedule
    n = O.theta_count(sched)
    assert H.theta_count(sched) == n
    seed = w.theta_seed if schedule is None else w.theta_seed + 7
    return W.draw_theta(n, w.theta_sigma, seed)


@functools.lru_cache(maxsize=None)
def plans(name: str, schedule=None, sign_offset=0):
    """(library plan, oracle transform) for a workload's schedule."""
    w = W.get(name)
    sched = schedule or w.schedule
    d = int(np.prod(sched))
    theta = theta_for(w, schedule)
    sign = w.sign_seed + sign_offset
    if w.theta_kind == "i8":
        codes, scales = W.quantize_theta_int8(theta, O.stage_theta_counts(sched))
        gp = H.Plan(d, sched, codes=codes, scales=scales, sign_seed=sign)
        op = O.make_plan(d, sched, codes=codes, scales=scales, sign_seed=sign)
    else:
        gp = H.Plan(d, sched, theta=theta, sign_seed=sign)
        op = O.make_plan(d, sched, theta, sign_seed=sign)
    gp.materialize()
    return gp, O.Transform(op)


@functools.lru_cache(maxsize=4)
def full_input(name: str, rows: int):
    return W.draw_encoded(W.get(name), 0, rows)


def check(enc_out, y_oracle, x_rows_f64, what):
    xn = np.linalg.norm(x_rows_f64, axis=1)
    if enc_out.dtype == np.uint16:
        return check_bf16(enc_out, y_oracle, xn, O.round_bf16, what)
    return check_f32(enc_out, y_oracle, xn, what)


def run(gp, enc, direction):
    x = to_dev(enc)
    y = gp.apply(x, direction=direction)
    torch.cuda.synchronize()
    return to_host(y)


# ---------------------------------------------------------------- workloads ---

@pytest.mark.parametrize("direction", ["forward", "inverse"])
def test_d64_fp32_full(direction):
    gp, tr = plans("d64")
    enc = full_input("d64", 1024)
    out = run(gp, enc, direction)
    check(out, tr.apply(decode(enc), direction), decode(enc), f"d64 {direction}")


def test_d64_hadamard_theta_zero_is_randomized_hadamard():
    import scipy.linalg
    gp, tr = plans("d64_hadamard")
    enc = full_input("d64_hadamard", 1024)
    out = run(gp, enc, "forward")
    x = decode(enc)
    check(out, tr.forward(x), x, "d64_hadamard vs oracle")
    want = (x * O.sign_vector(64, W.get("d64_hadamard").sign_seed)) @ scipy.linalg.hadamard(64).T / 8.0
    check(out, want, x, "d64_hadamard vs H_64 S")


@pytest.mark.parametrize("name,direction", [
    ("d4096", "forward"), ("d4096", "inverse"), ("d5120", "forward"), ("d5120", "inverse"),
    ("d8192_int8", "forward"), ("d8192_int8", "inverse")])
@pytest.mark.parametrize("rows", [1, 3, 37, 1000])
def test_small_batches_full_compare(name, direction, rows):
    gp, tr = plans(name)
    enc = W.draw_encoded(W.get(name), 0, rows)
    out = run(gp, enc, direction)
    check(out, tr.apply(decode(enc), direction), decode(enc), f"{name} {direction} rows={rows}")


@pytest.mark.parametrize("name,rows,direction", [
    ("d4096", 65536, "forward"),
    ("d5120", 32768, "forward"), ("d5120", 32768, "inverse"),
    ("d5120_64k", 65536, "forward"), ("d5120_64k", 65536, "inverse"),
    ("d8192_int8", 65536, "forward"), ("d8192_int8", 65536, "inverse"),
    ("d8192_int8", 256, "forward"), ("d8192_int8", 16, "inverse")])
def test_full_size_sampled(name, rows, direction):
    gp, tr = plans(name)
    enc = full_input(name, rows)
    out = run(gp, enc, direction)
    idx = W.sample_rows(rows, 768)
    x = decode(enc[idx])
    stats = check(out[idx], tr.apply(x, direction), x, f"{name} {direction} {rows} rows")
    # every row, not only the sampled ones: the transform is orthogonal, so the row
    # norm survives up to the bf16 rounding of input and output
    y_all = decode(out)
    nx = np.linalg.norm(decode(enc), axis=1)
    ny = np.linalg.norm(y_all, axis=1)
    assert np.all(np.abs(ny - nx) <= 2 ** -7 * nx + 1e-30), name
    assert np.isfinite(y_all).all()
    print(name, direction, rows, stats)


def test_d8192_int8_decode_rows_one():
    gp, tr = plans("d8192_int8")
    enc = full_input("d8192_int8", 1)
    for direction in ("forward", "inverse"):
        out = run(gp, enc, direction)
        check(out, tr.apply(decode(enc), direction), decode(enc), f"d8192_int8 rows=1 {direction}")


def test_round_trip_fp32_on_device():
    gp, _ = plans("d5120")
    x = torch.randn(300, 5120, device=DEV, dtype=torch.float32)
    y = gp.apply(x, direction="forward")
    z = gp.apply(y, direction="inverse")
    err = (z - x).abs().amax(dim=1) / x.norm(dim=1)
    assert float(err.max()) < 4e-6
    assert torch.allclose(y.norm(dim=1), x.norm(dim=1), rtol=2e-6)


# ---------------------------------------------------------------- two-sided ---

def _two_sided_plans(u_sched, v_sched, w):
    pu, tu = plans(w.name, tuple(u_sched), 11)
    pv, tv = plans(w.name, tuple(v_sched), 0)
    return pu, tu, pv, tv


def test_two_sided_small_full_compare():
    w = W.get("two_sided")
    pu, tu, pv, tv = _two_sided_plans((8, 8, 7), (8, 8, 2), w)
    wt = W.draw_encoded(w, 0, 448, 128)
    out = H.apply_two_sided(pu, pv, to_dev(wt))
    torch.cuda.synchronize()
    wf = decode(wt)
    want = tu.inverse(tv.inverse(wf).T).T                  # T_U^T W T_V
    got = to_host(out)
    tau = np.max(np.linalg.norm(wf, axis=1))
    check_bf16(got, want, np.full(got.shape[0], tau), O.round_bf16, "two-sided small")


def test_two_sided_full_size_sampled_rows():
    """C4 at full size (28672 x 8192): 448 output rows against the oracle, one in every 64-row
    slab (the column kernel's second pass) with the offsets inside the slab running through all
    64 residues seven times (so every 448-row set {p + 64 v} of its first pass is hit), plus the
    first and last rows."""
    w = W.get("two_sided")
    pu, tu, pv, tv = _two_sided_plans(w.u_schedule, w.schedule, w)
    wt = W.draw_encoded(w, 0, w.n_out, w.n_in)
    out = to_host(H.apply_two_sided(pu, pv, to_dev(wt)))
    torch.cuda.synchronize()
    k = np.arange(w.n_out // 64)
    rows = np.unique(np.concatenate([64 * k + (k % 64), W.sample_rows(w.n_out, 6)]))
    assert np.unique(rows // 64).size == w.n_out // 64 and np.unique(rows % 64).size == 64
    # row i of T_U^T W T_V is (T_U e_i)^T W T_V
    e = np.zeros((rows.size, w.n_out))
    e[np.arange(rows.size), rows] = 1.0
    u_cols = tu.forward(e)                                  # rows: (T_U e_i)^T
    wf = decode(wt)
    z = u_cols @ wf
    want = tv.inverse(z)
    tau = np.max(np.linalg.norm(wf, axis=1))
    stats = check_bf16(out[rows], want, np.full(rows.size, tau), O.round_bf16, "two-sided full")
    print("two-sided", stats)
    assert np.isfinite(decode(out)).all()
    # Frobenius norm is preserved by the two orthogonal factors
    nf = np.linalg.norm(wf)
    assert abs(np.linalg.norm(decode(out)) - nf) <= 2 ** -7 * nf


def test_two_sided_in_place():
    w = W.get("two_sided")
    pu, tu, pv, tv = _two_sided_plans((8, 8, 7), (8, 8, 2), w)
    wt = W.draw_encoded(w, 0, 448, 128)
    t = to_dev(wt)
    ref = to_host(H.apply_two_sided(pu, pv, t.clone()))
    H.apply_two_sided(pu, pv, t, t)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(to_host(t), ref)


# --------------------------------------------------------------- edge cases ---

def test_rows_zero_is_a_no_op():
    gp, _ = plans("d4096")
    x = torch.empty(0, 4096, device=DEV, dtype=torch.bfloat16)
    y = gp.apply(x)
    assert y.shape == (0, 4096)


@pytest.mark.parametrize("name", ["d4096", "d64"])
def test_in_place(name):
    gp, tr = plans(name)
    enc = W.draw_encoded(W.get(name), 0, 129)
    x = to_dev(enc)
    gp.apply(x, x)
    torch.cuda.synchronize()
    check(to_host(x), tr.forward(decode(enc)), decode(enc), f"{name} in place")


@pytest.mark.parametrize("name,pad", [("d4096", 3), ("d4096", 8), ("d64", 1), ("d5120", 16)])
def test_leading_dimension_and_guard_bands(name, pad):
    gp, tr = plans(name)
    w = W.get(name)
    rows, d = 70, w.d
    ld = d + pad
    enc = W.draw_encoded(w, 0, rows)
    canary = 0x7FC1 if enc.dtype == np.uint16 else np.float32(-123.25)
    buf_x = np.full(rows * ld + 64, canary, dtype=enc.dtype)
    buf_x[:rows * ld].reshape(rows, ld)[:, :d] = enc
    buf_y = np.full(rows * ld + 64, canary, dtype=enc.dtype)
    tx, ty = to_dev(buf_x), to_dev(buf_y)
    xv = tx[:rows * ld].view(rows, ld)[:, :d]
    yv = ty[:rows * ld].view(rows, ld)[:, :d]
    gp.apply(xv, yv)
    torch.cuda.synchronize()
    got = to_host(ty)
    body = got[:rows * ld].reshape(rows, ld)
    check(np.ascontiguousarray(body[:, :d]), tr.forward(decode(enc)), decode(enc), f"{name} ld={ld}")
    if enc.dtype == np.uint16:
        assert np.all(body[:, d:] == canary) and np.all(got[rows * ld:] == canary)
    else:
        assert np.all(body[:, d:] == canary) and np.all(got[rows * ld:] == canary)
    np.testing.assert_array_equal(to_host(tx), buf_x)      # input untouched


def test_two_streams_share_a_plan():
    gp, tr = plans("d4096")
    a = W.draw_encoded(W.get("d4096"), 0, 512)
    b = W.draw_encoded(W.get("d4096"), 512, 512)
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    xa, xb = to_dev(a), to_dev(b)
    torch.cuda.synchronize()
    with torch.cuda.stream(s1):
        ya = gp.apply(xa)
    with torch.cuda.stream(s2):
        yb = gp.apply(xb)
    torch.cuda.synchronize()
    check(to_host(ya), tr.forward(decode(a)), decode(a), "stream 1")
    check(to_host(yb), tr.forward(decode(b)), decode(b), "stream 2")


def test_partial_overlap_rejected():
    gp, _ = plans("d4096")
    buf = torch.zeros(8 * 4096 + 4096, device=DEV, dtype=torch.bfloat16)
    x = buf[:8 * 4096].view(8, 4096)
    y = buf[4096:].view(8, 4096)
    with pytest.raises(HB.HarpError) as e:
        gp.apply(x, y)
    assert e.value.status == HB.HARP_ERR_INVALID_ARG


def test_materialize_is_idempotent_and_blocks_are_reused():
    gp, tr = plans("d64")
    gp.materialize()
    enc = full_input("d64", 1024)
    out = run(gp, enc, "forward")
    check(out, tr.forward(decode(enc)), decode(enc), "after second materialize")


def test_bench_shape_uses_the_specialized_kernel_and_no_wait_gave_up():
    gp, tr = plans("d4096")
    enc = W.draw_encoded(W.get("d4096"), 0, 4096 + 5)
    out = run(gp, enc, "forward")
    assert H.last_kernel() == "harp_fast_d4096_fwd_kernel"
    gp.device_status()
    idx = W.sample_rows(enc.shape[0], 300)
    x = decode(enc[idx])
    check(out[idx], tr.forward(x), x, "fast kernel 4101 rows")

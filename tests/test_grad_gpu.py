"""GPU parity of the calibration backward (harp_grad_theta: dL/dtheta for
L = sum_r g_r . (T x_r), HARP technical summary §2.3 Optimization Objective) against the
float64 oracle on the same seeded rows and upstream gradients, for every workload schedule
on batches of several tiles with a ragged tail; the stationarity of L at g = T x at the
full C2 size (a property that holds at any size); edge cases and argument errors.

Tolerance.  The kernel keeps the stage chain in fp32: every value of z_t and h_t carries
at most about 2 m b_max u of its row's norm in rounding error (u = 2^-24; m stage
applications each way, b_max-term dot products), and the sums over rows add ntiles u of
the sum of the terms.  An entry of dL/dB_{t,c} is a sum of products h[k] z[l], so its
error is at most 2 eps sum_r |g_r| |x_r| with eps = 2 m b_max u + ntiles u, and a
parameter's gradient (two entries of dL/dA, |M| <= 1, |Q + I| <= 2) at most 8 times
that: the element-wise bound below.  Rounding errors are not all of one sign, so the
error taken over all parameters together is far below that worst case; the aggregate
check allows a relative l2 error of 2e-5."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H
from structured_rotations_b200 import harp as HB
from tests.test_parity_gpu import DEV, plans, to_dev, decode

pytestmark = pytest.mark.gpu
U = 2.0 ** -24


def _oracle_plan(name):
    return plans(name)[1].plan


def _check(got, x, g, op, what, ntiles):
    want = O.theta_grad(op, x, g)
    eps = 2 * op.m * max(op.schedule) * U + ntiles * U
    bound = 8 * eps * float(np.sum(np.linalg.norm(x, axis=1) * np.linalg.norm(g, axis=1)))
    err = np.abs(got.astype(np.float64) - want)
    k = int(np.argmax(err))
    assert err[k] <= bound, f"{what}: |dtheta - oracle| = {err[k]:.3e} at {k} > {bound:.3e}"
    rel = np.linalg.norm(err) / np.linalg.norm(want)
    assert rel <= 2e-5, f"{what}: relative l2 error {rel:.3e}"
    return rel


def _tile_rows(d):
    # rows per tile of the gradient kernel: two fp32 rows of d rounded up to 32 floats
    # within 227 KiB, at most 16
    rs = (d + 31) // 32 * 32
    return min(16, (227 * 1024) // (8 * rs))


@pytest.mark.parametrize("name,rows", [("d64", 37), ("d64_hadamard", 53), ("d4096", 23), ("d5120", 19),
                                       ("d8192_int8", 11)])
def test_grad_theta_vs_oracle(name, rows):
    gp, tr = plans(name)
    w = W.get(name)
    xe, ge = W.draw_encoded(w, 0, rows), W.draw_upstream(w, 0, rows)
    dth = gp.grad_theta(to_dev(xe), to_dev(ge))
    torch.cuda.synchronize()
    assert H.last_kernel() == "harp_grad_blocks_kernel"
    ntiles = -(-rows // _tile_rows(w.d))
    assert ntiles >= 2
    _check(dth.cpu().numpy(), decode(xe), decode(ge), tr.plan, f"{name} rows={rows}", ntiles)


@pytest.mark.parametrize("schedule", [(5, 2, 8), (7, 8), (3, 4, 2), (6, 6), (2, 2, 2, 2, 2, 2, 2)])
def test_grad_theta_other_radices_fp32(schedule):
    d = int(np.prod(schedule))
    theta = W.draw_theta(O.theta_count(schedule), 0.3, 23)
    gp = H.Plan(d, schedule, theta=theta, sign_seed=9).materialize()
    op = O.make_plan(d, schedule, theta.astype(np.float32).astype(np.float64), sign_seed=9)
    rng = np.random.default_rng(d)
    rows = 3 * _tile_rows(d) + 5
    x = rng.standard_normal((rows, d)).astype(np.float32)
    g = rng.standard_normal((rows, d)).astype(np.float32)
    dth = gp.grad_theta(to_dev(x), to_dev(g))
    torch.cuda.synchronize()
    _check(dth.cpu().numpy(), x.astype(np.float64), g.astype(np.float64), op, f"{schedule}", 4)


def test_grad_theta_padded_and_unaligned_rows_and_empty_batch():
    gp, tr = plans("d64")
    w = W.get("d64")
    xe, ge = W.draw_encoded(w, 0, 40), W.draw_upstream(w, 0, 40)
    xp = torch.zeros(40, 80, dtype=torch.float32, device=DEV)
    gq = torch.zeros(40, 65, dtype=torch.float32, device=DEV)     # rows not 16-byte aligned: scalar loads
    xp[:, :64] = to_dev(xe)
    gq[:, :64] = to_dev(ge)
    dth = gp.grad_theta(xp[:, :64], gq[:, :64])
    torch.cuda.synchronize()
    _check(dth.cpu().numpy(), decode(xe), decode(ge), tr.plan, "padded", 3)
    empty = torch.empty(0, 64, dtype=torch.float32, device=DEV)
    out = torch.full((H.theta_count(w.schedule),), 7.0, device=DEV)
    gp.grad_theta(empty, empty, out)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0


def test_grad_theta_argument_errors():
    gp, _ = plans("d64")
    x = torch.zeros(4, 64, dtype=torch.float32, device=DEV)
    n = H.theta_count((8, 8))
    out = torch.empty(n, dtype=torch.float32, device=DEV)
    ws = torch.empty(HB.lib().harp_grad_workspace_bytes(gp.handle) - 16, dtype=torch.uint8, device=DEV)
    with pytest.raises(HB.HarpError) as e:
        gp.grad_theta(x, x, out, ws)
    assert e.value.status == HB.HARP_ERR_INVALID_ARG
    big = H.Plan(32, (16, 2), sign_seed=1).materialize()          # radix above 8
    with pytest.raises(HB.HarpError) as e:
        big.grad_theta(torch.zeros(2, 32, device=DEV), torch.zeros(2, 32, device=DEV))
    assert e.value.status == HB.HARP_ERR_UNSUPPORTED
    fresh = H.Plan(64, (8, 8), sign_seed=1)                        # not materialized
    with pytest.raises(HB.HarpError) as e:
        fresh.grad_theta(x, x)
    assert e.value.status == HB.HARP_ERR_NOT_MATERIALIZED


def test_full_size_gradient_vanishes_at_the_stationary_point():
    """C2 size (65,536 rows, d = 4096), fp32 rows: with g = T x the loss is at its maximum
    over theta (sum_r <T x_r, T' x_r> <= sum_r |x_r|^2), so dL/dtheta = 0 up to rounding;
    against the gradient for upstream rows of the same norms in random directions."""
    gp, _ = plans("d4096")
    w = W.get("d4096")
    rows = 65536
    x = to_dev(W.draw_encoded(w, 0, rows)).float()
    y = gp.apply(x)
    gen = torch.Generator(device=DEV).manual_seed(5)
    g_rand = torch.randn(rows, w.d, generator=gen, device=DEV)
    g_rand *= (y.norm(dim=1) / g_rand.norm(dim=1)).unsqueeze(1)
    d_stat = gp.grad_theta(x, y)
    d_rand = gp.grad_theta(x, g_rand)
    torch.cuda.synchronize()
    ratio = (d_stat.abs().max() / d_rand.abs().max()).item()
    assert ratio < 1e-3, ratio

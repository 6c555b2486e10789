"""GPU parity of the moment check that picks the number of composed passes
(harp_moment_check; the RHT-composition page's linear-time check on the input's moments, read
as the per-row moments m2, m3, m4 and the peakedness m4 / m2^2 against two caller thresholds)
against the float64 oracle.  The kernel squares and sums in double, so the moments agree with
the oracle's to summation order (relative 1e-12), and the pass counts agree wherever a row's
peakedness is not within that of a threshold."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from oracle import harp_oracle as O
import workloads as W
import structured_rotations_b200 as H

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dev(vals, dtype, pad=0):
    rows, d = vals.shape
    full = np.zeros((rows, d + pad))
    full[:, :d] = vals
    if dtype == "bf16":
        t = torch.from_numpy(W.encode_bf16(full).view(np.int16)).view(torch.bfloat16).to(DEV)
    else:
        t = torch.from_numpy(full.astype(np.float32)).to(DEV)
    return t[:, :d]


def _stored(x, dtype):
    return W.decode_bf16(W.encode_bf16(x)) if dtype == "bf16" else x.astype(np.float32).astype(np.float64)


@pytest.mark.parametrize("rows,d,dtype,pad", [(300, 4096, "bf16", 0), (65, 5120, "f32", 0), (33, 8192, "bf16", 8),
                                               (17, 100, "f32", 3), (5, 7, "bf16", 0)])
def test_moments_and_passes_match_the_oracle(rows, d, dtype, pad):
    rng = np.random.default_rng([rows, d])
    x = rng.standard_t(3, size=(rows, d))
    x[0] = 0.0                                           # a zero row
    x[1] = 0.0
    x[1, d // 2] = 2.5                                   # a one-hot row
    x[2] = 1.0                                           # a flat row
    x[3:, rng.choice(d, min(8, d), replace=False)] *= 50.0   # outlier channels
    vals = _stored(x, dtype)
    m, k = H.moment_check(_dev(vals, dtype, pad), 4.0 / d, 40.0 / d)
    torch.cuda.synchronize()
    want = O.row_moments(vals)
    np.testing.assert_allclose(m.cpu().numpy(), want, rtol=1e-12, atol=0)
    kap = O.peakedness(want)
    ref = O.passes_needed(kap, 4.0 / d, 40.0 / d)
    near = (np.abs(kap - 4.0 / d) < 1e-12 * kap) | (np.abs(kap - 40.0 / d) < 1e-12 * kap)
    got = k.cpu().numpy()
    assert np.all((got == ref) | near)
    assert got[0] == 1 and got[2] == 1                  # zero and flat rows: one pass
    if d >= 64:
        assert got[1] == 3                              # a one-hot row: kappa = 1 > 40 / d


def test_one_pass_of_the_rotation_lowers_the_needed_passes():
    """Rows with heavy outlier channels (the d = 4096 workload) need more passes than the same
    rows after one rotation through the library."""
    w = W.get("d4096")
    theta = W.draw_theta(O.theta_count(w.schedule), w.theta_sigma, w.theta_seed)
    gp = H.Plan(w.d, w.schedule, theta=theta, sign_seed=w.sign_seed).materialize()
    enc = W.draw_encoded(w, 0, 512)
    x = torch.from_numpy(enc.view(np.int16)).view(torch.bfloat16).to(DEV)
    tau1, tau2 = 4.0 / w.d, 40.0 / w.d
    _, before = H.moment_check(x, tau1, tau2)
    _, after = H.moment_check(gp.apply(x), tau1, tau2)
    torch.cuda.synchronize()
    b, a = before.cpu().numpy(), after.cpu().numpy()
    assert b.mean() > a.mean()
    assert np.all(a <= b)


def test_one_theta_zero_pass_flattens_one_hot_rows():
    """At theta = 0 the rotation is a randomized Hadamard transform: a one-hot row comes out flat
    (peakedness exactly 1/d), so it needs one pass after it and three before."""
    d, sched = 4096, (8, 8, 8, 8)
    gp = H.Plan(d, sched, sign_seed=9).materialize()
    x = torch.zeros(64, d, dtype=torch.float32, device=DEV)
    x[torch.arange(64), torch.arange(64) * 61] = 1.0
    m0, k0 = H.moment_check(x, 4.0 / d, 40.0 / d)
    m1, k1 = H.moment_check(gp.apply(x), 4.0 / d, 40.0 / d)
    torch.cuda.synchronize()
    m0, m1 = m0.cpu().numpy(), m1.cpu().numpy()
    np.testing.assert_allclose(O.peakedness(m0), 1.0, rtol=0)
    np.testing.assert_allclose(O.peakedness(m1), 1.0 / d, rtol=1e-6)
    assert k0.cpu().numpy().tolist() == [3] * 64 and k1.cpu().numpy().tolist() == [1] * 64

"""Pins of the oracle's moment check (the RHT-composition page: a linear-time check on the
input's moments picks the number of composed passes; the statistic is read as the per-row
moments m2, m3, m4, the peakedness m4 / m2^2 and the Berry-Esseen ratio m3 / m2^(3/2)).
Fixed by closed forms: a one-hot row has peakedness and ratio 1; a flat row 1/d and d^-1/2;
both are invariant under scaling and sign flips and lie between those extremes (Hoelder);
one theta = 0 pass of an all-power-of-two schedule turns a one-hot row into a flat one, so
its peakedness drops from 1 to exactly 1/d."""
import numpy as np
import pytest

from oracle import harp_oracle as O


def test_one_hot_and_flat_rows():
    d = 64
    x = np.zeros((2, d))
    x[0, 17] = -3.0
    x[1, :] = 0.5
    m = O.row_moments(x)
    assert m[0].tolist() == [9.0, 27.0, 81.0]
    assert m[1].tolist() == [d * 0.25, d * 0.125, d * 0.0625]
    k = O.peakedness(m)
    r = O.berry_esseen_ratio(m)
    assert k[0] == 1.0 and r[0] == 1.0
    assert k[1] == pytest.approx(1 / d, rel=1e-15) and r[1] == pytest.approx(d ** -0.5, rel=1e-15)


def test_zero_row():
    m = O.row_moments(np.zeros((1, 8)))
    assert m.tolist() == [[0.0, 0.0, 0.0]]
    assert O.peakedness(m)[0] == 0.0 and O.berry_esseen_ratio(m)[0] == 0.0


def test_scale_and_sign_invariance_and_hoelder_bounds():
    rng = np.random.default_rng(5)
    x = rng.standard_t(3, size=(50, 256))
    m = O.row_moments(x)
    k, r = O.peakedness(m), O.berry_esseen_ratio(m)
    signs = np.where(rng.random(x.shape) < 0.5, -1.0, 1.0)
    m2 = O.row_moments(-7.5 * x * signs)
    np.testing.assert_allclose(O.peakedness(m2), k, rtol=1e-13)
    np.testing.assert_allclose(O.berry_esseen_ratio(m2), r, rtol=1e-13)
    d = x.shape[1]
    assert np.all(k >= 1 / d - 1e-15) and np.all(k <= 1 + 1e-15)
    assert np.all(r >= d ** -0.5 - 1e-15) and np.all(r <= 1 + 1e-15)
    # Cauchy-Schwarz: m3 = sum |x| x^2 <= sqrt(sum x^2) sqrt(sum x^4), so m3^2 <= m2 m4
    assert np.all(m[:, 1] ** 2 <= m[:, 0] * m[:, 2] * (1 + 1e-13))


def test_gaussian_rows_have_peakedness_near_three_over_d():
    rng = np.random.default_rng(6)
    d = 4096
    k = O.peakedness(O.row_moments(rng.standard_normal((200, d))))
    assert abs(k.mean() * d - 3.0) < 0.05


@pytest.mark.parametrize("schedule", [(8, 8), (2, 2, 2, 2, 2, 2), (4, 8, 2)])
def test_one_theta_zero_pass_flattens_a_one_hot_row(schedule):
    d = int(np.prod(schedule))
    tr = O.Transform(O.make_plan(d, schedule, None, sign_seed=3))
    x = np.zeros((d, d))
    x[np.arange(d), np.arange(d)] = 1.0
    k0 = O.peakedness(O.row_moments(x))
    k1 = O.peakedness(O.row_moments(tr.forward(x)))
    assert np.all(k0 == 1.0)
    np.testing.assert_allclose(k1, 1 / d, rtol=1e-12)


def test_passes_needed_thresholds():
    k = np.array([0.0, 0.01, 0.02, 0.05, 0.5, 1.0])
    assert O.passes_needed(k, 0.01, 0.05).tolist() == [1, 1, 2, 2, 3, 3]

"""Pins of the oracle's composition of rotations (T = T_{k-1} ... T_0, plans[0] first):
at theta = 0 with power-of-two radices every factor is the normalized Sylvester Hadamard
times its signs, so the composite is the product of those matrices (scipy's Hadamard
routine); orthogonality; the inverse is the transpose; the order of the factors matters."""
import numpy as np
import scipy.linalg

from oracle import harp_oracle as O


def _tr(schedule, sign_seed, scale=0.0, seed=0):
    d = int(np.prod(schedule))
    theta = np.random.default_rng(seed).standard_normal(O.theta_count(schedule)) * scale
    return O.Transform(O.make_plan(d, schedule, theta, sign_seed=sign_seed))


def test_theta_zero_composite_is_a_product_of_signed_hadamards():
    h = scipy.linalg.hadamard(64) / 8.0
    parts = [_tr((8, 8), 5), _tr((2, 2, 2, 2, 2, 2), 6), _tr((4, 16), 7)]
    c = O.Composed(parts)
    want = np.eye(64)
    for s in (5, 6, 7):
        want = h @ np.diag(O.sign_vector(64, s)) @ want
    np.testing.assert_allclose(c.forward(np.eye(64)).T, want, atol=1e-12)


def test_composite_is_orthogonal_and_inverse_is_transpose():
    c = O.Composed([_tr((8, 5, 2), 1, 0.4, 1), _tr((2, 5, 8), 2, 0.4, 2), _tr((5, 8, 2), 3, 0.4, 3)])
    t = c.forward(np.eye(80)).T
    np.testing.assert_allclose(t.T @ t, np.eye(80), atol=1e-12)
    x = np.random.default_rng(0).standard_normal((4, 80))
    np.testing.assert_allclose(c.inverse(c.forward(x)), x, atol=1e-12)
    np.testing.assert_allclose(c.inverse(np.eye(80)).T, t.T, atol=1e-12)


def test_factor_order_matters():
    a, b = _tr((8, 8), 1, 0.3, 1), _tr((8, 8), 2, 0.3, 2)
    x = np.random.default_rng(1).standard_normal((3, 64))
    np.testing.assert_allclose(O.Composed([a, b]).forward(x), b.forward(a.forward(x)), atol=1e-12)
    assert np.max(np.abs(O.Composed([a, b]).forward(x) - O.Composed([b, a]).forward(x))) > 1e-3

"""Pins of the oracle's calibration backward (dL/dtheta for L = sum_r g_r . (T x_r),
HARP technical summary §2.3 Optimization Objective: theta is fitted from calibration
data, so the fit needs this gradient).  Each pin is fixed by something other than the
oracle's own chain rule: central finite differences of the oracle's forward transform,
closed forms of one-stage transforms at theta = 0 and for Givens rotations, the
stationarity of L at g = T x, and additivity over rows."""
import math

import numpy as np
import pytest

from oracle import harp_oracle as O


def _plan(schedule, scale, seed, sign_seed=3):
    d = int(np.prod(schedule))
    theta = np.random.default_rng(seed).standard_normal(O.theta_count(schedule)) * scale
    return O.make_plan(d, schedule, theta, sign_seed=sign_seed)


def _loss(plan, theta, x, g):
    p = O.make_plan(plan.d, plan.schedule, theta, sign_seed=plan.sign_seed, qr_seed=plan.qr_seed)
    return float(np.sum(g * O.Transform(p).forward(x)))


@pytest.mark.parametrize("schedule", [(8, 8), (2, 2, 2, 2, 2, 2), (5, 2, 8), (7, 8), (3, 4), (6,)])
def test_theta_grad_matches_central_differences(schedule):
    plan = _plan(schedule, 0.3, sum(schedule))
    rng = np.random.default_rng(7)
    x = rng.standard_normal((4, plan.d))
    g = rng.standard_normal((4, plan.d))
    got = O.theta_grad(plan, x, g)
    h = 1e-6
    # every parameter for the smaller schedules, an even spread of 60 for the larger
    ks = range(plan.theta.size) if plan.theta.size <= 120 else np.linspace(0, plan.theta.size - 1, 60).astype(int)
    for k in ks:
        e = np.zeros_like(plan.theta)
        e[k] = h
        fd = (_loss(plan, plan.theta + e, x, g) - _loss(plan, plan.theta - e, x, g)) / (2 * h)
        assert abs(fd - got[k]) <= 1e-6 * (1 + abs(got[k])), (schedule, k, fd, got[k])


@pytest.mark.parametrize("b", [3, 4, 8])
def test_one_stage_cayley_gradient_at_zero_closed_form(b):
    # d = b, one stage, theta = 0: T = G S, and Q = I + 2A + O(A^2), so
    # dL/dtheta_k = 2 (g_i v_j - g_j v_i) with v = G S x for the k-th pair (i < j) in
    # row-major order of the strict upper triangle
    plan = O.make_plan(b, (b,), np.zeros(O.theta_count((b,))), sign_seed=11)
    rng = np.random.default_rng(b)
    x, g = rng.standard_normal((1, b)), rng.standard_normal((1, b))
    v = O.base_mixer(b) @ (O.sign_vector(b, 11) * x[0])
    want = [2 * (g[0, i] * v[j] - g[0, j] * v[i]) for i in range(b) for j in range(i + 1, b)]
    np.testing.assert_allclose(O.theta_grad(plan, x, g), want, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("theta", [0.0, 0.7, -2.5])
def test_one_stage_givens_gradient_closed_form(theta):
    # d = 2: L = g . (R(theta) v), v = G_2 S x, dR/dtheta = [[-sin, -cos], [cos, -sin]]
    plan = O.make_plan(2, (2,), np.array([theta]), sign_seed=5)
    x, g = np.array([[0.3, -1.2]]), np.array([[0.8, 0.25]])
    v = O.base_mixer(2) @ (O.sign_vector(2, 5) * x[0])
    c, s = math.cos(theta), math.sin(theta)
    want = g[0] @ np.array([[-s, -c], [c, -s]]) @ v
    np.testing.assert_allclose(O.theta_grad(plan, x, g), [want], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("schedule", [(8, 8), (5, 2, 8), (2, 2, 2, 2, 2, 2)])
def test_gradient_vanishes_where_the_loss_is_stationary(schedule):
    # with g_r = T x_r, L(theta') = sum_r <T x_r, T' x_r> <= sum_r |x_r|^2 with equality at
    # theta' = theta, so theta is a maximum and the gradient is zero
    plan = _plan(schedule, 0.5, 3)
    x = np.random.default_rng(1).standard_normal((6, plan.d))
    g = O.Transform(plan).forward(x)
    got = O.theta_grad(plan, x, g)
    assert np.max(np.abs(got)) <= 1e-12 * np.sum(x * x)


def test_gradient_is_additive_over_rows():
    plan = _plan((8, 5, 2), 0.4, 9)
    rng = np.random.default_rng(2)
    x, g = rng.standard_normal((7, plan.d)), rng.standard_normal((7, plan.d))
    whole = O.theta_grad(plan, x, g)
    parts = O.theta_grad(plan, x[:3], g[:3]) + O.theta_grad(plan, x[3:], g[3:])
    np.testing.assert_allclose(whole, parts, rtol=1e-12, atol=1e-12)


def test_gradient_scale_bounds_the_gradient():
    plan = _plan((8, 8), 0.4, 4)
    rng = np.random.default_rng(3)
    x, g = rng.standard_normal((5, plan.d)), rng.standard_normal((5, plan.d))
    assert np.all(np.abs(O.theta_grad(plan, x, g)) <= 4 * O.theta_grad_scale(plan, x, g) + 1e-12)

"""Pins of the oracle's fit terms on a Hessian proxy (HARP technical summary §2.3: L_fit =
L_diag + lambda_bd R_bd, described in words only; the readings are in the oracle).  Fixed by
invariants and closed forms: a block-diagonal matrix has no off-block energy; a multiple of
the identity stays one under any rotation; a constant matrix has off-block energy 1 - q/n;
rotation keeps the total energy; L_diag vanishes on weights the quantizer represents
exactly, equals the plain squared error for H = I, scales with the square of the weight and
is bounded by a quarter step squared per entry."""
import numpy as np
import pytest
import scipy.linalg

from oracle import harp_oracle as O


def _plan(schedule, seed, scale=0.3):
    d = int(np.prod(schedule))
    theta = np.random.default_rng(seed).standard_normal(O.theta_count(schedule)) * scale
    return O.make_plan(d, schedule, theta, sign_seed=seed + 1)


def _spd(n, seed):
    a = np.random.default_rng(seed).standard_normal((n, 2 * n))
    return a @ a.T / (2 * n)


def test_block_diagonal_has_no_off_block_energy():
    blocks = [_spd(8, s) for s in range(4)]
    assert O.off_block_energy(scipy.linalg.block_diag(*blocks), 8) == 0.0
    assert O.off_block_energy(scipy.linalg.block_diag(*blocks), 32) == 0.0
    assert O.off_block_energy(scipy.linalg.block_diag(*blocks), 4) > 0.0


def test_constant_matrix_closed_form():
    for n, q in ((64, 8), (64, 32), (80, 16)):
        assert O.off_block_energy(np.ones((n, n)), q) == pytest.approx(1 - q / n, abs=1e-15)


@pytest.mark.parametrize("schedule", [(8, 8), (5, 2, 8), (2, 2, 2, 2, 2, 2)])
def test_identity_proxy_stays_block_diagonal_under_rotation(schedule):
    plan = _plan(schedule, 3)
    d = plan.d
    assert O.r_bd(plan, 2.5 * np.eye(d), 8 if d % 8 == 0 else 4) < 1e-28


@pytest.mark.parametrize("schedule", [(8, 8), (5, 2, 8)])
def test_rotation_keeps_total_energy_and_spd(schedule):
    plan = _plan(schedule, 5)
    h = _spd(plan.d, 7)
    hr = O.rotated_hessian(plan, h)
    assert np.sum(hr * hr) == pytest.approx(np.sum(h * h), rel=1e-12)
    np.testing.assert_allclose(hr, hr.T, atol=1e-12)
    assert np.min(np.linalg.eigvalsh(hr)) > 0
    t = O.Transform(plan).dense()
    np.testing.assert_allclose(hr, t.T @ h @ t, atol=1e-12)


def test_l_diag_vanishes_on_exact_weights_and_scales_quadratically():
    rng = np.random.default_rng(2)
    codes = rng.integers(-127, 128, size=(6, 64))
    codes[:, ::32] = 127                                   # every block reaches the full scale
    s = np.exp(rng.standard_normal((6, 2)))
    w = (codes.reshape(6, 2, 32) * s[..., None]).reshape(6, 64)
    h = _spd(64, 4)
    assert O.l_diag(w, h, 32) < 1e-20 * np.sum(w * w)
    w2 = rng.standard_normal((6, 64))
    assert O.l_diag(4.0 * w2, h, 32) == pytest.approx(16.0 * O.l_diag(w2, h, 32), rel=1e-12)


def test_l_diag_with_identity_proxy_is_the_squared_error_and_bounded():
    rng = np.random.default_rng(3)
    w = rng.standard_normal((5, 128))
    q, s = O.quantize_blocks(w, 64)
    target = (q.reshape(5, 2, 64) * s[..., None]).reshape(5, 128)
    assert O.l_diag(w, np.eye(128), 64) == pytest.approx(np.sum((w - target) ** 2), rel=1e-12)
    assert O.l_diag(w, np.eye(128), 64) <= np.sum((np.repeat(s, 64, axis=1) / 2) ** 2)

"""Pins for the float64 oracle: each check ties a part of it to something other
than itself (published values, library routines, closed forms, invariants, an
independent restatement), so that a dropped term, a wrong sign or index, or a
transposed operand anywhere in it fails at least one test.  CPU only."""
import math
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.stats

from oracle import harp_oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if line:
                rows.append(line.split())
    return rows


def _rand_plan(d, schedule, seed, sigma=0.3, sign_seed=11):
    rng = np.random.default_rng(seed)
    theta = sigma * rng.standard_normal(O.theta_count(schedule))
    return O.make_plan(d, schedule, theta, sign_seed=sign_seed)


# --------------------------------------------------------------------- RNG ---

def test_splitmix64_published_outputs():
    want = [int(r[0], 16) for r in _read_golden("splitmix64_seed0.txt")]
    assert O.splitmix64(0, len(want)) == want


def test_unit_double_range():
    us = O.splitmix64(12345, 4096)
    vals = [O.unit_double(u) for u in us]
    assert min(vals) >= 0.0 and max(vals) < 1.0
    assert O.unit_double((1 << 64) - 1) == 1.0 - 2.0 ** -53
    assert O.unit_double(0) == 0.0


def test_gaussian_matrix_is_standard_normal():
    g = O.gaussian_matrix(300, 777).ravel()          # 90,000 draws
    assert abs(g.mean()) < 0.02
    assert abs(g.var() - 1.0) < 0.02
    assert scipy.stats.kstest(g, "norm").pvalue > 1e-3


def test_sign_vector_balanced_and_deterministic():
    s = O.sign_vector(8192, 3002)
    assert set(np.unique(s)) == {-1.0, 1.0}
    assert abs(s.mean()) < 0.05
    np.testing.assert_array_equal(s, O.sign_vector(8192, 3002))
    assert not np.array_equal(s, O.sign_vector(8192, 3003))


# ----------------------------------------------------------- base mixers ---

@pytest.mark.parametrize("b", [1, 2, 4, 8, 16, 32])
def test_sylvester_matches_scipy_hadamard(b):
    np.testing.assert_array_equal(O.sylvester_mixer(b) * math.sqrt(b),
                                  scipy.linalg.hadamard(b).astype(float))


@pytest.mark.parametrize("b", [3, 5, 6, 7, 12])
def test_qr_mixer_is_the_positive_diagonal_qr(b):
    g = O.qr_mixer(b)
    m = O.gaussian_matrix(b, O.QR_SEED_BASE + b)
    np.testing.assert_allclose(g.T @ g, np.eye(b), atol=1e-14)
    r = g.T @ m                                   # M = G R  =>  R = G^T M
    np.testing.assert_allclose(np.tril(r, -1), 0.0, atol=1e-13)
    assert np.all(np.diag(r) > 0)


def test_qr_seed_selects_a_different_mixer():
    assert not np.allclose(O.qr_mixer(5), O.qr_mixer(5, qr_seed=99))
    assert O.base_mixer(8).shape == (8, 8) and np.allclose(O.base_mixer(8), O.sylvester_mixer(8))


# ------------------------------------------------------ learnable factor ---

def test_givens_group_law_and_orientation():
    a, b = 0.37, -1.21
    np.testing.assert_allclose(O.givens(a) @ O.givens(b), O.givens(a + b), atol=1e-15)
    np.testing.assert_allclose(O.givens(math.pi / 2) @ np.array([1.0, 0.0]), [0.0, 1.0], atol=1e-15)
    assert abs(np.linalg.det(O.givens(0.9)) - 1.0) < 1e-15


@pytest.mark.parametrize("b", [3, 4, 5, 7, 8])
@pytest.mark.parametrize("scale", [0.05, 1.0, 3.0])
def test_cayley_orthogonal_det_plus_one(b, scale):
    rng = np.random.default_rng(b * 100 + int(scale * 10))
    q = O.cayley(scale * rng.standard_normal(O.params_per_block(b)), b)
    np.testing.assert_allclose(q.T @ q, np.eye(b), atol=1e-12)
    assert abs(np.linalg.det(q) - 1.0) < 1e-12


@pytest.mark.parametrize("a", [0.0, 0.2, -0.7, 2.5])
def test_cayley_b2_closed_form(a):
    want = np.array([[1 - a * a, 2 * a], [-2 * a, 1 - a * a]]) / (1 + a * a)
    np.testing.assert_allclose(O.cayley([a], 2), want, atol=1e-15)
    np.testing.assert_allclose(O.cayley([a], 2), O.givens(-2 * math.atan(a)), atol=1e-15)


def test_cayley_parameter_order_block_diagonal():
    # strict upper triangle, row-major: (0,1)->0, (2,3)->13, (4,5)->22, (6,7)->27
    a = [0.3, -0.8, 1.7, 0.05]
    p = np.zeros(28)
    p[[0, 13, 22, 27]] = a
    want = scipy.linalg.block_diag(*[O.givens(-2 * math.atan(v)) for v in a])
    np.testing.assert_allclose(O.cayley(p, 8), want, atol=1e-14)


def test_cayley_series():
    rng = np.random.default_rng(5)
    p = 1e-4 * rng.standard_normal(28)
    a = O.skew_from_params(p, 8)
    # (I - A)^{-1} (I + A) = I + 2A + 2A^2 + 2A^3 + O(A^4)
    approx = np.eye(8) + 2 * a + 2 * a @ a
    np.testing.assert_allclose(O.cayley(p, 8), approx, atol=1e-10)
    np.testing.assert_allclose(O.cayley(p, 8), approx + 2 * a @ a @ a, atol=1e-14)
    assert np.allclose(a, -a.T) and a[0, 1] == p[0] and a[1, 2] == p[7]


# ------------------------------------------------------- layout / counts ---

@pytest.mark.parametrize("schedule,want", [
    ((8, 8), 448), ((2,) * 6, 192), ((8, 8, 8, 8), 57344), ((8, 8, 8, 5, 2), 66560),
    ((8, 8, 8, 8, 2), 118784), ((8, 8, 8, 8, 7), 487424)])
def test_theta_counts_closed_form(schedule, want):
    d = int(np.prod(schedule))
    assert O.theta_count(schedule) == want == d * sum(b - 1 for b in schedule) // 2


def test_int8_storage_overhead_matches_reported_bits_per_weight():
    # 2-bit 7B: int8 theta on both sides of a 4096 x 4096 layer, radix-8 blocks
    per_side = O.theta_count((8, 8, 8, 8))
    extra_bits = 2 * per_side * 8 / 4096 ** 2
    assert abs(extra_bits - 0.05) < 0.01       # reported 2.00 -> 2.05 bits/param


def test_int8_dequantize_and_encoder_error():
    sched = (8, 8, 8, 5, 2)
    theta = W.draw_theta(O.theta_count(sched), math.sqrt(0.05), 9)
    codes, scales = W.quantize_theta_int8(theta, O.stage_theta_counts(sched))
    deq = O.dequantize_int8(codes, scales, sched)
    off = 0
    for t, n in enumerate(O.stage_theta_counts(sched)):
        assert np.all(np.abs(deq[off:off + n] - theta[off:off + n]) <= scales[t] * 0.5 + 1e-12)
        assert deq[off + 3] == float(codes[off + 3]) * float(scales[t])
        off += n


# --------------------------------------------------------------- stages ---

def _tensor_forward(plan, x):
    """Independent restatement: view x as a tensor with one axis per digit
    (digit 0 last) and contract stage t's blocks against axis t, with the block
    index running over the remaining digits in mixed-radix order."""
    sched = plan.schedule
    m = len(sched)
    blocks = O.stage_blocks(plan)
    z = (x * O.sign_vector(plan.d, plan.sign_seed)).reshape(tuple(reversed(sched)))
    for t, b in enumerate(sched):
        ax = m - 1 - t
        other = tuple(sched[j] for j in reversed(range(m)) if j != t)
        bt = blocks[t].reshape(other + (b, b))
        zt = np.moveaxis(z, ax, -1)
        zt = np.einsum("...kl,...l->...k", bt, zt)
        z = np.moveaxis(zt, -1, ax)
    return z.reshape(plan.d)


@pytest.mark.parametrize("schedule", [(8, 8), (5, 2, 8), (3, 4, 2), (2, 3, 5, 2), (7, 8), (8, 5)])
def test_sparse_stages_match_tensor_restatement(schedule):
    d = int(np.prod(schedule))
    plan = _rand_plan(d, schedule, seed=d)
    x = np.random.default_rng(1).standard_normal(d)
    np.testing.assert_allclose(O.apply(plan, x[None, :])[0], _tensor_forward(plan, x), atol=1e-13)


@pytest.mark.parametrize("schedule", [(2,) * 6, (8, 8), (4, 4, 4), (2, 8, 4)])
def test_theta_zero_power_of_two_is_sylvester_hadamard_times_signs(schedule):
    plan = O.make_plan(64, schedule, None, sign_seed=3001)
    t = O.Transform(plan).dense()
    want = scipy.linalg.hadamard(64) / 8.0 * O.sign_vector(64, 3001)[None, :]
    np.testing.assert_allclose(t, want, atol=1e-14)


@pytest.mark.parametrize("schedule", [(8, 5, 2), (5, 2, 8), (7, 8), (3, 5)])
def test_theta_zero_mixed_radix_is_kronecker_of_mixers(schedule):
    d = int(np.prod(schedule))
    plan = O.make_plan(d, schedule, None, sign_seed=5)
    k = np.ones((1, 1))
    for b in schedule:                 # G_{b_{m-1}} (x) ... (x) G_{b_0}
        k = np.kron(O.base_mixer(b), k)
    want = k * O.sign_vector(d, 5)[None, :]
    np.testing.assert_allclose(O.Transform(plan).dense(), want, atol=1e-13)


@pytest.mark.parametrize("schedule", [(8, 8), (2,) * 6, (5, 2, 8), (7, 8), (8, 5), (4, 3, 5), (2, 2, 7)])
def test_dense_transform_is_orthogonal(schedule):
    d = int(np.prod(schedule))
    assert d <= 256
    t = O.Transform(_rand_plan(d, schedule, seed=3, sigma=0.8)).dense()
    np.testing.assert_allclose(t.T @ t, np.eye(d), atol=1e-13)


def test_inverse_is_transpose():
    tr = O.Transform(_rand_plan(40, (5, 2, 4), seed=8))
    inv = tr.inverse(np.eye(40)).T
    np.testing.assert_allclose(inv, tr.dense().T, atol=1e-14)


@pytest.mark.parametrize("schedule", [(8, 8, 8, 8), (8, 8, 8, 5, 2)])
def test_norm_preservation_and_round_trip(schedule):
    d = int(np.prod(schedule))
    tr = O.Transform(_rand_plan(d, schedule, seed=4, sigma=0.22))
    x = np.random.default_rng(2).standard_normal((4, d)) * 7.0
    y = tr.forward(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    np.testing.assert_allclose(tr.inverse(y), x, atol=1e-12 * np.abs(x).max())


def test_theta_zero_transform_equals_randomized_hadamard_on_rows():
    plan = O.make_plan(4096, (8, 8, 8, 8), None, sign_seed=3)
    x = np.random.default_rng(3).standard_normal((2, 4096))
    want = (x * O.sign_vector(4096, 3)) @ scipy.linalg.hadamard(4096).T / 64.0
    np.testing.assert_allclose(O.apply(plan, x), want, atol=1e-12)


def test_two_sided_matches_dense_matrices():
    pu = _rand_plan(12, (4, 3), seed=21, sign_seed=1)
    pv = _rand_plan(10, (5, 2), seed=22, sign_seed=2)
    w = np.random.default_rng(0).standard_normal((12, 10))
    tu, tv = O.Transform(pu).dense(), O.Transform(pv).dense()
    np.testing.assert_allclose(O.two_sided(pu, pv, w), tu.T @ w @ tv, atol=1e-13)
    # and the change of basis is exact: W = T_U W_out T_V^T
    np.testing.assert_allclose(tu @ O.two_sided(pu, pv, w) @ tv.T, w, atol=1e-13)


# ------------------------------------------------------------ rounding ---

def test_round_bf16_hand_worked_values():
    for src, want in _read_golden("bf16_rne.txt"):
        x = float.fromhex(src)
        assert O.round_bf16(np.array([x]))[0] == float.fromhex(want), src


def test_round_bf16_agrees_with_input_encoder():
    rng = np.random.default_rng(0)
    x = rng.standard_normal(200000) * np.exp(rng.uniform(-30, 30, 200000))
    np.testing.assert_array_equal(O.round_bf16(x), W.decode_bf16(W.encode_bf16(x)))


def test_round_bf16_is_nearest():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(10000)
    r = O.round_bf16(x)
    m, e = np.frexp(x)
    ulp = np.ldexp(1.0, e - 8)
    assert np.all(np.abs(r - x) <= ulp / 2)


def test_hand_worked_blocks_pin_the_factor_order():
    # B = Q(theta) G: Hadamard preconditioning first, learnable factor second.
    # radix 2, theta = pi/2: Q = [[0,-1],[1,0]], G = [[1,1],[1,-1]]/sqrt2
    #   Q G = [[-1, 1], [1, 1]] / sqrt2      (G Q would be [[1,-1],[-1,-1]] / sqrt2)
    plan = O.make_plan(2, (2,), [math.pi / 2], sign_seed=0)
    np.testing.assert_allclose(O.stage_blocks(plan)[0][0],
                               np.array([[-1.0, 1.0], [1.0, 1.0]]) / math.sqrt(2), atol=1e-15)
    # radix 4, only A[0][1] = 1: Cayley gives Givens(-pi/2) on plane (0,1),
    # Q = [[0,1,0,0],[-1,0,0,0],[0,0,1,0],[0,0,0,1]]; rows of Q G are
    # (G row 1, -G row 0, G row 2, G row 3) with G = H_4 / 2
    theta = np.zeros(O.theta_count((4,)))
    theta[0] = 1.0
    plan = O.make_plan(4, (4,), theta, sign_seed=0)
    want = np.array([[1, -1, 1, -1], [-1, -1, -1, -1], [1, 1, -1, -1], [1, -1, -1, 1]]) / 2.0
    np.testing.assert_allclose(O.stage_blocks(plan)[0][0], want, atol=1e-15)

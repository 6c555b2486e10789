"""HARP rotation oracle: a plain, slow, float64 CPU restatement of the transform.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA library (no kernels, headers, tables or helpers) and never calls it.

What it computes (sources are the HARP pages: "Technical Summary: HARP
(Hadamard-Preconditioned Adaptive Rotation Processor)", gist.science, and its
Chinese twin; the arXiv abstract "HARP: Hadamard-Preconditioned Adaptive
Rotation Processor for Extreme LLM Quantization"):

* §2.1 Core Architecture: a mixed-radix schedule b = (b_0..b_{m-1}) with
  prod b_t = d; stage t applies a block-diagonal orthogonal matrix to groups of
  b_t coordinates separated by stride permutations.
* §2.2 Hadamard Preconditioning: every block is B_{t,c}(theta) = Q_{t,c}(theta) G_{b_t};
  G is the normalized Sylvester Hadamard for powers of two, else the QR of a fixed
  Gaussian matrix; Q is a Givens rotation for b=2 and a Cayley map for b>2;
  theta = 0 gives Q = I and the fixed randomized Hadamard transform.
* §2.4 Deployment Efficiency: theta may be stored as int8.
* Abstract: a two-sided processor (one rotation on each side of a weight).

Readings taken where the pages leave a step open (each is also listed in the
design notes):

* digit order: index i = sum_t i_t s_t with s_t = prod_{j<t} b_j (digit 0 least
  significant); stage t mixes digit t; block index c = lo + s_t*hi with
  lo = i mod s_t, hi = i div (s_t b_t).
* order: y = M_{m-1} ... M_1 M_0 S x (random signs first, stage 0 next).
* S: s_i = -1 if the top bit of the i-th SplitMix64 output of the sign seed is
  set, else +1.
* G_b (b not a power of two): one matrix per radix value; entries row-major from
  a SplitMix64 stream seeded with (qr_seed or 0x4841525000000000) + b; each
  entry consumes two outputs u1, u2 mapped to U = (u >> 11) 2^-53 and
  g = sqrt(-2 ln(1-U1)) cos(2 pi U2); G = Q diag(sign R_kk) from M = QR, sign(0)=+1.
* G_b (power of two): G[k][l] = (-1)^popcount(k & l) / sqrt(b).
* Givens: Q(theta) = [[cos, -sin], [sin, cos]].
* Cayley: A[i][j] = theta_k for i<j in row-major order of the strict upper
  triangle, A[j][i] = -theta_k, Q = (I - A)^{-1} (I + A); one parameter set per block.
* theta layout: stages in order; within a stage, blocks in c order; p_t
  parameters per block (1 for b=2, b(b-1)/2 otherwise).
* int8 theta: theta = q * scale_t, one float32 scale per stage.
* two-sided: W_out = T_U^T W T_V (rows of W take the inverse V transform, columns
  the inverse U transform).

Pins (tests/test_oracle_pins.py): SplitMix64 published outputs, Gaussian
statistics, scipy's Sylvester Hadamard, the unique positive-diagonal QR, Givens
group law, Cayley orthogonality / det +1 / closed forms, theta=0 Kronecker form,
an independent tensor-axis restatement of the stages, dense orthogonality,
round trips and bf16 rounding of hand-worked values.

Beyond the forward transform, three parts that build on it (each with its own pins):
the calibration backward dL/dtheta (§2.3; tests/test_oracle_grad_pins.py: central
differences, one-stage closed forms, stationarity, additivity), the blockwise int8
quantizer of the rotated rows (§2.4; tests/test_oracle_quant_pins.py: hand-worked
codes, zero blocks, the half-step bound, scaling) and the composition of rotations
(tests/test_oracle_compose_pins.py: the theta = 0 product of signed Hadamards,
orthogonality, inverse, factor order).  The fit's evaluation terms R_bd and L_diag
(tests/test_oracle_fit_pins.py: invariants and closed forms only) and the moment check that
picks the number of composed passes (tests/test_oracle_moment_pins.py: one-hot and flat
rows, scale invariance, Hoelder bounds, a one-hot row flattened by one theta = 0 pass).
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np
import scipy.sparse as sp

MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15
QR_SEED_BASE = 0x4841525000000000  # "HARP" in the top four bytes


# ---------------------------------------------------------------------------
# SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom number
# generators", OOPSLA 2014; the 64-bit finalizer of Vigna's reference code)
# ---------------------------------------------------------------------------

def splitmix64(seed: int, n: int) -> List[int]:
    """The first n outputs of the SplitMix64 stream whose state starts at seed."""
    state = seed & MASK64
    out = []
    for _ in range(n):
        state = (state + GOLDEN_GAMMA) & MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
        out.append(z ^ (z >> 31))
    return out


def unit_double(u: int) -> float:
    """Top 53 bits of a 64-bit output as a double in [0, 1)."""
    return (u >> 11) * 2.0 ** -53


def sign_vector(d: int, sign_seed: int) -> np.ndarray:
    """The random +-1 diagonal S of the randomized Hadamard transform."""
    return np.array([-1.0 if (u >> 63) else 1.0 for u in splitmix64(sign_seed, d)])


def gaussian_matrix(b: int, seed: int) -> np.ndarray:
    """b x b standard normal entries, row-major, Box-Muller cosine branch."""
    u = splitmix64(seed, 2 * b * b)
    g = np.empty(b * b)
    for e in range(b * b):
        u1 = unit_double(u[2 * e])
        u2 = unit_double(u[2 * e + 1])
        g[e] = math.sqrt(-2.0 * math.log(1.0 - u1)) * math.cos(2.0 * math.pi * u2)
    return g.reshape(b, b)


# ---------------------------------------------------------------------------
# Base mixers G_b (§2.2 "G_{b_t} is a fixed base mixer")
# ---------------------------------------------------------------------------

def is_pow2(b: int) -> bool:
    return b >= 1 and (b & (b - 1)) == 0


def sylvester_mixer(b: int) -> np.ndarray:
    """Normalized Sylvester Hadamard: entry (k, l) is (-1)^popcount(k & l) / sqrt(b)."""
    g = np.empty((b, b))
    for k in range(b):
        for l in range(b):
            g[k, l] = -1.0 if bin(k & l).count("1") % 2 else 1.0
    return g / math.sqrt(b)


def qr_mixer(b: int, qr_seed: int = 0) -> np.ndarray:
    """Deterministic orthogonal fallback: Q factor of a fixed seeded Gaussian
    matrix, columns signed so that R has a non-negative diagonal."""
    base = qr_seed if qr_seed else QR_SEED_BASE
    m = gaussian_matrix(b, (base + b) & MASK64)
    q, r = np.linalg.qr(m)
    sgn = np.where(np.diag(r) < 0, -1.0, 1.0)
    return q * sgn[None, :]


def base_mixer(b: int, qr_seed: int = 0) -> np.ndarray:
    return sylvester_mixer(b) if is_pow2(b) else qr_mixer(b, qr_seed)


# ---------------------------------------------------------------------------
# Learnable factor Q_{t,c}(theta) (§2.2)
# ---------------------------------------------------------------------------

def params_per_block(b: int) -> int:
    return 1 if b == 2 else b * (b - 1) // 2


def givens(theta: float) -> np.ndarray:
    c, s = math.cos(theta), math.sin(theta)
    return np.array([[c, -s], [s, c]])


def skew_from_params(params: Sequence[float], b: int) -> np.ndarray:
    a = np.zeros((b, b))
    k = 0
    for i in range(b):
        for j in range(i + 1, b):
            a[i, j] = params[k]
            a[j, i] = -params[k]
            k += 1
    return a


def cayley(params: Sequence[float], b: int) -> np.ndarray:
    a = skew_from_params(params, b)
    eye = np.eye(b)
    return np.linalg.solve(eye - a, eye + a)


def learnable_factor(params: Sequence[float], b: int) -> np.ndarray:
    if b == 2:
        return givens(float(params[0]))
    return cayley(params, b)


# ---------------------------------------------------------------------------
# Plan: schedule, strides, theta layout
# ---------------------------------------------------------------------------

@dataclasses.dataclass
class OraclePlan:
    d: int
    schedule: tuple
    theta: np.ndarray                 # float64, concatenated per stage/block
    sign_seed: int
    qr_seed: int = 0

    def __post_init__(self):
        self.schedule = tuple(int(b) for b in self.schedule)
        if int(np.prod(self.schedule)) != self.d:
            raise ValueError("product of the schedule must equal d")
        self.theta = np.asarray(self.theta, dtype=np.float64)
        if self.theta.size != theta_count(self.schedule):
            raise ValueError("theta has the wrong length for this schedule")

    @property
    def m(self) -> int:
        return len(self.schedule)


def strides(schedule: Sequence[int]) -> List[int]:
    s, out = 1, []
    for b in schedule:
        out.append(s)
        s *= b
    return out


def stage_theta_counts(schedule: Sequence[int]) -> List[int]:
    d = int(np.prod(schedule))
    return [(d // b) * params_per_block(b) for b in schedule]


def theta_count(schedule: Sequence[int]) -> int:
    return sum(stage_theta_counts(schedule))


def dequantize_int8(codes: np.ndarray, scales: np.ndarray, schedule: Sequence[int]) -> np.ndarray:
    """int8 storage (§2.4): theta = q * scale_t in float64."""
    out = np.empty(codes.size)
    off = 0
    for t, n in enumerate(stage_theta_counts(schedule)):
        out[off:off + n] = codes[off:off + n].astype(np.float64) * float(scales[t])
        off += n
    return out


def make_plan(d, schedule, theta=None, sign_seed=0, qr_seed=0, codes=None, scales=None) -> OraclePlan:
    if codes is not None:
        theta = dequantize_int8(np.asarray(codes), np.asarray(scales), schedule)
    if theta is None:
        theta = np.zeros(theta_count(schedule))
    return OraclePlan(int(d), tuple(schedule), np.asarray(theta, dtype=np.float64),
                      int(sign_seed), int(qr_seed))


# ---------------------------------------------------------------------------
# Blocks B_{t,c} = Q_{t,c}(theta) G_{b_t} and explicit sparse stage matrices
# ---------------------------------------------------------------------------

def stage_blocks(plan: OraclePlan) -> List[np.ndarray]:
    """Per stage, an array [d/b_t, b_t, b_t] holding B_{t,c}[k][l] (k out, l in)."""
    blocks = []
    off = 0
    for b in plan.schedule:
        g = base_mixer(b, plan.qr_seed)
        p = params_per_block(b)
        nb = plan.d // b
        bt = np.empty((nb, b, b))
        for c in range(nb):
            q = learnable_factor(plan.theta[off + c * p: off + (c + 1) * p], b)
            bt[c] = q @ g
        off += nb * p
        blocks.append(bt)
    return blocks


def stage_matrix(d: int, b: int, s: int, blocks_t: np.ndarray) -> sp.csr_matrix:
    """M_t with M_t[lo + s(k + b hi), lo + s(l + b hi)] = B_{t,c}[k][l], c = lo + s hi."""
    rows, cols, vals = [], [], []
    for c in range(d // b):
        lo, hi = c % s, c // s
        for k in range(b):
            for l in range(b):
                rows.append(lo + s * (k + b * hi))
                cols.append(lo + s * (l + b * hi))
                vals.append(blocks_t[c, k, l])
    return sp.csr_matrix((vals, (rows, cols)), shape=(d, d))


def stage_matrices(plan: OraclePlan) -> List[sp.csr_matrix]:
    blocks = stage_blocks(plan)
    return [stage_matrix(plan.d, b, s, blocks[t])
            for t, (b, s) in enumerate(zip(plan.schedule, strides(plan.schedule)))]


class Transform:
    """T = M_{m-1} ... M_0 S for one plan, with its stage matrices built once."""

    def __init__(self, plan: OraclePlan):
        self.plan = plan
        self.signs = sign_vector(plan.d, plan.sign_seed)
        self.mats = stage_matrices(plan)

    def forward(self, x: np.ndarray) -> np.ndarray:
        """y = T x for every row x of a [rows, d] array."""
        z = np.asarray(x, dtype=np.float64) * self.signs[None, :]
        for mt in self.mats:
            z = (mt @ z.T).T
        return z

    def inverse(self, y: np.ndarray) -> np.ndarray:
        """x = T^T y = S M_0^T ... M_{m-1}^T y for every row."""
        z = np.asarray(y, dtype=np.float64)
        for mt in reversed(self.mats):
            z = (mt.T @ z.T).T
        return z * self.signs[None, :]

    def apply(self, x: np.ndarray, direction: str) -> np.ndarray:
        if direction == "forward":
            return self.forward(x)
        if direction == "inverse":
            return self.inverse(x)
        raise ValueError(direction)

    def dense(self) -> np.ndarray:
        """T itself, built column by column from the unit vectors."""
        return self.forward(np.eye(self.plan.d)).T


def apply(plan: OraclePlan, x: np.ndarray, direction: str = "forward") -> np.ndarray:
    return Transform(plan).apply(x, direction)


def two_sided(plan_u: OraclePlan, plan_v: OraclePlan, w: np.ndarray) -> np.ndarray:
    """W_out = T_U^T W T_V for W of shape [d_U, d_V] (abstract: two-sided processor)."""
    tv = Transform(plan_v)
    tu = Transform(plan_u)
    z = tv.inverse(np.asarray(w, dtype=np.float64))      # rows: w_r^T T_V = (T_V^T w_r)^T
    return tu.inverse(z.T).T                             # columns: T_U^T col


# ---------------------------------------------------------------------------
# Output rounding to the I/O dtype
# ---------------------------------------------------------------------------

def round_bf16(x: np.ndarray) -> np.ndarray:
    """Nearest bf16 value (8 significant bits, ties to even) of each float64,
    rounded directly from float64; returned as float64."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m 2^e, 0.5 <= |m| < 1
    normal = np.ldexp(np.rint(m * 256.0), e - 8)
    sub = np.rint(x * 2.0 ** 133) * 2.0 ** -133   # below 2^-126: fixed spacing 2^-133
    return np.where(np.abs(x) < 2.0 ** -126, sub, normal)


def round_f32(x: np.ndarray) -> np.ndarray:
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# Calibration backward: the gradient of a loss with respect to theta
# ---------------------------------------------------------------------------
#
# HARP is fitted per layer from calibration data by minimizing a surrogate loss
# (§2.3 Optimization Objective), so a fit needs dL/dtheta through the transform.
# For rows x_r with upstream gradients g_r = dL/dy_r of y_r = T x_r, the loss is
# locally L = sum_r g_r . (T x_r) and its gradient is built here from the chain
# rule, step by step:
#
#   z_0 = S x, z_{t+1} = M_t z_t        (stage inputs, forward)
#   h_m = g,   h_t = M_t^T h_{t+1}      (gradients at the stage inputs, backward)
#   dL/dB_{t,c}[k][l] = sum_r h_{t+1,r}[lo + s_t (k + b_t hi)] z_{t,r}[lo + s_t (l + b_t hi)]
#   dL/dQ = dL/dB G^T                   (B = Q G)
#   Givens: dL/dtheta = sum dL/dQ * dQ/dtheta, dQ/dtheta = [[-sin, -cos], [cos, -sin]]
#   Cayley: Q = M (I + A) with M = (I - A)^{-1}, so dQ = M dA (Q + I) and
#           dL/dA = M^T dL/dQ (Q + I)^T; theta_k sits at A[i][j] = theta_k and
#           A[j][i] = -theta_k, so dL/dtheta_k = dL/dA[i][j] - dL/dA[j][i].
#
# dL/dx itself is T^T g, the inverse transform.  For int8 storage the gradient is
# taken with respect to the dequantized values q * scale_t.

def block_grads(plan: OraclePlan, x: np.ndarray, g: np.ndarray) -> List[np.ndarray]:
    """dL/dB_{t,c} for L = sum_r g_r . (T x_r): per stage an array [d/b_t, b_t, b_t]."""
    tr = Transform(plan)
    z = np.asarray(x, dtype=np.float64) * tr.signs[None, :]
    inputs = []
    for mt in tr.mats:
        inputs.append(z)
        z = (mt @ z.T).T
    h = np.asarray(g, dtype=np.float64)
    out = [None] * plan.m
    for t in reversed(range(plan.m)):
        b, s = plan.schedule[t], strides(plan.schedule)[t]
        zt = inputs[t]
        gb = np.zeros((plan.d // b, b, b))
        for c in range(plan.d // b):
            lo, hi = c % s, c // s
            idx = [lo + s * (k + b * hi) for k in range(b)]
            gb[c] = h[:, idx].T @ zt[:, idx]          # sum over rows of h[k] z[l]
        out[t] = gb
        h = (tr.mats[t].T @ h.T).T
    return out


def theta_grad_from_blocks(plan: OraclePlan, dblocks: List[np.ndarray]) -> np.ndarray:
    """dL/dtheta from dL/dB_{t,c} through B = Q(theta) G (Givens or Cayley)."""
    out = np.empty(theta_count(plan.schedule))
    off = 0
    for t, b in enumerate(plan.schedule):
        g = base_mixer(b, plan.qr_seed)
        p = params_per_block(b)
        for c in range(plan.d // b):
            par = plan.theta[off + c * p: off + (c + 1) * p]
            dq = dblocks[t][c] @ g.T
            if b == 2:
                cs, sn = math.cos(par[0]), math.sin(par[0])
                out[off + c] = np.sum(dq * np.array([[-sn, -cs], [cs, -sn]]))
            else:
                a = skew_from_params(par, b)
                eye = np.eye(b)
                minv = np.linalg.inv(eye - a)
                q = minv @ (eye + a)
                da = minv.T @ dq @ (q + eye).T
                k = 0
                for i in range(b):
                    for j in range(i + 1, b):
                        out[off + c * p + k] = da[i, j] - da[j, i]
                        k += 1
        off += (plan.d // b) * p
    return out


def theta_grad(plan: OraclePlan, x: np.ndarray, g: np.ndarray) -> np.ndarray:
    """dL/dtheta for L = sum_r g_r . (T(theta) x_r), in the theta layout of the plan."""
    return theta_grad_from_blocks(plan, block_grads(plan, x, g))


def theta_grad_scale(plan: OraclePlan, x: np.ndarray, g: np.ndarray) -> np.ndarray:
    """Per parameter, sum_r |h_{t+1,r}[group]| |z_{t,r}[group]| over the rows for the
    parameter's block: every entry of dL/dB_{t,c} is at most this in magnitude, and
    |dL/dtheta| at most 4 times it (|M| <= 1, |Q + I| <= 2, G orthogonal, two entries
    per parameter).  Used to scale comparison tolerances."""
    tr = Transform(plan)
    z = np.asarray(x, dtype=np.float64) * tr.signs[None, :]
    inputs = []
    for mt in tr.mats:
        inputs.append(z)
        z = (mt @ z.T).T
    h = np.asarray(g, dtype=np.float64)
    per_stage = [None] * plan.m
    for t in reversed(range(plan.m)):
        b, s = plan.schedule[t], strides(plan.schedule)[t]
        zt = inputs[t]
        sc = np.zeros(plan.d // b)
        for c in range(plan.d // b):
            lo, hi = c % s, c // s
            idx = [lo + s * (k + b * hi) for k in range(b)]
            sc[c] = np.sum(np.linalg.norm(h[:, idx], axis=1) * np.linalg.norm(zt[:, idx], axis=1))
        per_stage[t] = sc
        h = (tr.mats[t].T @ h.T).T
    return np.concatenate([np.repeat(per_stage[t], params_per_block(b)) for t, b in enumerate(plan.schedule)])


# ---------------------------------------------------------------------------
# Blockwise quantizer on the rotated rows (fused epilogue)
# ---------------------------------------------------------------------------
#
# HARP is a drop-in preprocessing step in front of a blockwise quantizer (§2.4
# Deployment Efficiency; §2.3: the fit targets the deployed blockwise quantizer), so
# the rotated rows are quantized right away.  The quantizer here is the plain
# symmetric round-to-nearest one: per aligned block of qblock coordinates of a row,
# s = max |y| / 127 and q = clamp(round_half_even(y / s), -127, 127); s = 0 and
# q = 0 for an all-zero block.

def quantize_blocks(y: np.ndarray, qblock: int):
    """(int8 codes [rows, d], float64 scales [rows, d / qblock]) of rows y."""
    y = np.asarray(y, dtype=np.float64)
    rows, d = y.shape
    if d % qblock:
        raise ValueError("qblock must divide d")
    yb = y.reshape(rows, d // qblock, qblock)
    s = np.max(np.abs(yb), axis=2) / 127.0
    safe = np.where(s > 0, s, 1.0)
    q = np.where(s[..., None] > 0, np.rint(yb / safe[..., None]), 0.0)
    return np.clip(q, -127, 127).astype(np.int8).reshape(rows, d), s


# ---------------------------------------------------------------------------
# Composition of rotations
# ---------------------------------------------------------------------------
#
# Composing independent randomized Hadamard transforms brings every input's coordinates
# close to the behaviour of a uniform random rotation (the RHT-composition results the
# HARP pages quote: two passes for scalar quantization, three for vector quantization).
# The composite of plans P_0 .. P_{k-1} is T = T_{k-1} ... T_0 (P_0 acts first); its
# inverse is T_0^T ... T_{k-1}^T.

class Composed:
    """T = T_{k-1} ... T_1 T_0 for transforms of one dimension."""

    def __init__(self, transforms: Sequence[Transform]):
        if not transforms or len({t.plan.d for t in transforms}) != 1:
            raise ValueError("need transforms of one dimension")
        self.transforms = list(transforms)

    def forward(self, x: np.ndarray) -> np.ndarray:
        for t in self.transforms:
            x = t.forward(x)
        return x

    def inverse(self, y: np.ndarray) -> np.ndarray:
        for t in reversed(self.transforms):
            y = t.inverse(y)
        return y

    def apply(self, x: np.ndarray, direction: str) -> np.ndarray:
        if direction == "forward":
            return self.forward(x)
        if direction == "inverse":
            return self.inverse(x)
        raise ValueError(direction)


# ---------------------------------------------------------------------------
# The fit's evaluation terms on a Hessian proxy (§2.3 Optimization Objective)
# ---------------------------------------------------------------------------
#
# The pages describe the two terms of L_fit = L_diag + lambda_bd R_bd in words only; the
# readings here:
#  * the input-side Hessian proxy H (d_in x d_in, symmetric positive definite, e.g. X^T X of
#    calibration activations) in the rotated basis: inputs rotate as x' = T_V^T x, so
#    H' = T_V^T H T_V;
#  * R_bd: the energy of H' outside the diagonal blocks of the quantizer's block size q,
#    as a fraction of its total energy, sum_{I != J} |H'_IJ|_F^2 / |H'|_F^2;
#  * L_diag: the rotated weight W' = T_U^T W T_V against its blockwise target Q(W')
#    (the round-to-nearest int8 quantizer of quantize_blocks along the rows, dequantized),
#    each column j weighted by the diagonal of H': sum_j H'_jj sum_r (W'_rj - Q(W')_rj)^2.

def rotated_hessian(plan_v: OraclePlan, h: np.ndarray) -> np.ndarray:
    """H' = T_V^T H T_V."""
    tv = Transform(plan_v)
    z = tv.inverse(np.asarray(h, dtype=np.float64))      # rows: (T_V^T h_r)^T = h_r^T T_V
    return tv.inverse(z.T).T                             # columns: T_V^T (H T_V)


def off_block_energy(h: np.ndarray, q: int) -> float:
    """sum over blocks I != J of |H_IJ|_F^2 over |H|_F^2, blocks of q x q."""
    h = np.asarray(h, dtype=np.float64)
    n = h.shape[0]
    if h.shape != (n, n) or n % q:
        raise ValueError("square matrix with q dividing its size")
    total = float(np.sum(h * h))
    blk = np.arange(n) // q
    off = float(np.sum((h * h)[blk[:, None] != blk[None, :]]))   # summed directly, not total - diag
    return off / total if total > 0 else 0.0


def r_bd(plan_v: OraclePlan, h: np.ndarray, q: int) -> float:
    return off_block_energy(rotated_hessian(plan_v, h), q)


def l_diag(w_rot: np.ndarray, h_rot: np.ndarray, q: int) -> float:
    """sum_j H'_jj sum_r (W'_rj - Q(W')_rj)^2 for the rotated weight and Hessian proxy."""
    w = np.asarray(w_rot, dtype=np.float64)
    codes, scales = quantize_blocks(w, q)
    target = (codes.reshape(w.shape[0], -1, q) * scales[..., None]).reshape(w.shape)
    return float(np.sum(np.diag(h_rot)[None, :] * (w - target) ** 2))


# ---------------------------------------------------------------------------
# Moment check that picks the number of composed passes
# ---------------------------------------------------------------------------
#
# The RHT-composition page proposes a linear-time check on the input's moments that adapts at
# run time how many randomized Hadamard passes are applied, without giving the statistic or
# its thresholds.  Reading: one pass turns x into coordinates that are Rademacher-weighted sums
# of the entries of x, whose distance from a Gaussian is governed by how concentrated x is;
# the check computes, per row, the moments
#     m2 = sum x_i^2,  m3 = sum |x_i|^3,  m4 = sum x_i^4
# and from them the Berry-Esseen ratio rho = m3 / m2^(3/2) (in [d^-1/2, 1]) and the peakedness
# kappa = m4 / m2^2 (in [1/d, 1]: 1/d for a flat row, 1 for a one-hot row).  The number of
# passes is the smallest k in (1, 2, 3) whose threshold the row meets: kappa <= tau_1 -> 1,
# kappa <= tau_2 -> 2, else 3 (three for block (vector) quantizers in any case, per the page);
# the thresholds are the caller's.

def row_moments(x: np.ndarray) -> np.ndarray:
    """[rows, 3] float64: (sum x^2, sum |x|^3, sum x^4) of every row."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    return np.stack([np.sum(a * a, axis=1), np.sum(a * a * a, axis=1), np.sum((a * a) * (a * a), axis=1)], axis=1)


def peakedness(m: np.ndarray) -> np.ndarray:
    """kappa = m4 / m2^2 per row (0 for a zero row)."""
    m = np.asarray(m, dtype=np.float64)
    m2 = m[:, 0]
    return np.where(m2 > 0, m[:, 2] / np.where(m2 > 0, m2 * m2, 1.0), 0.0)


def berry_esseen_ratio(m: np.ndarray) -> np.ndarray:
    """rho = m3 / m2^(3/2) per row (0 for a zero row)."""
    m = np.asarray(m, dtype=np.float64)
    m2 = m[:, 0]
    return np.where(m2 > 0, m[:, 1] / np.where(m2 > 0, m2 ** 1.5, 1.0), 0.0)


def passes_needed(kappa: np.ndarray, tau1: float, tau2: float) -> np.ndarray:
    """The smallest number of passes (1, 2 or 3) whose threshold each row's kappa meets."""
    kappa = np.asarray(kappa, dtype=np.float64)
    return np.where(kappa <= tau1, 1, np.where(kappa <= tau2, 2, 3)).astype(np.int32)

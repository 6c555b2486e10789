"""Seeded synthetic inputs for the HARP rotation workloads.

Every array here is a pure function of (workload, seed, row range): rows are
drawn in blocks of ``ROW_BLOCK`` rows, each block from its own NumPy PCG64
stream keyed by ``[seed, block]``, so any sampled row of a 65,536-row batch can
be regenerated on its own without drawing the rest.

Workloads (HARP, "Technical Summary: HARP", sections 2.1-2.4; the shapes and
value distributions are the ones the five workload definitions name):

* ``d64``   d=64, schedule (8,8), 1024 rows fp32, x iid N(0,1), theta ~ N(0, 0.1)
* ``d64_hadamard``  d=64, schedule (2,2,2,2,2,2), theta = 0 (the fixed randomized Hadamard)
* ``d4096``   d=4096, (8,8,8,8), 65,536 rows bf16, Student-t (nu=3) entries with 8
           seeded outlier channels x50, theta ~ N(0, 0.05), forward
* ``d5120``   d=5120, (8,8,8,5,2), 32,768 rows bf16, N(0,1) with 1% of entries x20,
           theta ~ N(0, 0.05), forward and inverse (``d5120_64k``: 65,536 rows)
* ``two_sided``   two-sided U^T W V: W 28672x8192 bf16 iid N(0, 0.02^2) with 16 outlier
           columns x30; U (8,8,8,8,7), V (8,8,8,8,2), theta ~ N(0, 0.05)
* ``d8192_int8``   d=8192, (8,8,8,8,2), int8 theta + per-stage fp32 scale, bf16 rows in
           {1, 16, 256, 65536}, iid N(0,1), forward and inverse

"N(0, v)" is read as variance v (the same workload list writes the weight
distribution as N(0, 0.02^2)), so theta's standard deviation is sqrt(v).

Seeds: data = 1000 + k, theta = 2000 + k, sign seed = 3000 + k, where k is the
workload's seed index (1 for d64 and d64_hadamard, 2 for d4096, 3 for d5120 and
d5120_64k, 4 for two_sided, 5 for d8192_int8).
"""
from __future__ import annotations

import concurrent.futures as cf
import dataclasses
import math
import os
from typing import Optional, Sequence

import numpy as np

ROW_BLOCK = 256

__all__ = [
    "ROW_BLOCK", "Workload", "WORKLOADS", "get", "draw_rows", "draw_theta",
    "encode_bf16", "decode_bf16", "quantize_theta_int8", "sample_rows",
    "draw_weight", "draw_encoded", "draw_upstream", "C5_ROWS", "draw_hessian",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int                      # k in the seed recipe
    d: int
    schedule: tuple
    rows: int
    dtype: str                      # "f32" or "bf16"
    dist: str                       # value distribution of x
    theta_sigma: float              # standard deviation of theta (0 => theta = 0)
    theta_kind: str = "f32"         # "f32" or "i8"
    dirs: tuple = ("forward",)
    # two-sided only: the U plan (output side) and V plan (input side)
    u_schedule: Optional[tuple] = None
    n_out: int = 0
    n_in: int = 0

    @property
    def data_seed(self) -> int:
        return 1000 + self.index

    @property
    def theta_seed(self) -> int:
        return 2000 + self.index

    @property
    def sign_seed(self) -> int:
        return 3000 + self.index

    @property
    def io_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2


_S01 = math.sqrt(0.1)
_S005 = math.sqrt(0.05)

WORKLOADS = {
    "d64": Workload("d64", 1, 64, (8, 8), 1024, "f32", "normal", _S01,
                   dirs=("forward", "inverse")),
    "d64_hadamard": Workload("d64_hadamard", 1, 64, (2, 2, 2, 2, 2, 2), 1024, "f32", "normal", 0.0),
    "d4096": Workload("d4096", 2, 4096, (8, 8, 8, 8), 65536, "bf16", "student_t_outlier_channels",
                   _S005),
    "d5120": Workload("d5120", 3, 5120, (8, 8, 8, 5, 2), 32768, "bf16", "normal_sparse_x20",
                   _S005, dirs=("forward", "inverse")),
    "d5120_64k": Workload("d5120_64k", 3, 5120, (8, 8, 8, 5, 2), 65536, "bf16",
                       "normal_sparse_x20", _S005, dirs=("forward", "inverse")),
    # two-sided: rows of W get the V side (d = n_in), columns the U side (d = n_out)
    "two_sided": Workload("two_sided", 4, 8192, (8, 8, 8, 8, 2), 28672, "bf16", "weight_outlier_columns",
                   _S005, dirs=("two_sided",), u_schedule=(8, 8, 8, 8, 7),
                   n_out=28672, n_in=8192),
    "d8192_int8": Workload("d8192_int8", 5, 8192, (8, 8, 8, 8, 2), 65536, "bf16", "normal", _S005,
                   theta_kind="i8", dirs=("forward", "inverse")),
}

C5_ROWS = (1, 16, 256, 65536)


def get(name: str, rows: Optional[int] = None) -> Workload:
    w = WORKLOADS[name]
    if rows is not None:
        w = dataclasses.replace(w, rows=int(rows))
    return w


# ---------------------------------------------------------------------------
# bf16 storage format (bit patterns held as uint16)
# ---------------------------------------------------------------------------

def encode_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even) and return the bits.

    Rounds directly from float64 (no intermediate float32 rounding).  Values whose
    magnitude is below bf16's smallest normal are handled by scaling, so the
    result is correctly rounded there too.
    """
    x = np.asarray(x, dtype=np.float64)
    bits = np.array(x, dtype=np.float64, copy=True).view(np.uint64)
    # add half an ulp of the 7-bit mantissa (minus one) plus the lowest kept bit,
    # then clear the 45 dropped bits: round-to-nearest-even on the bit pattern
    lsb = bits >> np.uint64(45)
    lsb &= np.uint64(1)
    bits += lsb
    del lsb
    bits += np.uint64((1 << 44) - 1)
    bits &= ~np.uint64((1 << 45) - 1)
    f32 = bits.view(np.float64).astype(np.float32)
    del bits
    out = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    if x.size and np.abs(x).min() < 2.0 ** -126:
        tiny = (np.abs(x) < 2.0 ** -126) & (x != 0)
        t = np.rint(x[tiny] * 2.0 ** 133) * 2.0 ** -133
        out[tiny] = (t.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    return out


def decode_bf16(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float64."""
    b = np.asarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# activations / weights
# ---------------------------------------------------------------------------

def _outlier_columns(seed: int, d: int, count: int) -> np.ndarray:
    rng = np.random.default_rng([seed, 0x0C0])
    return np.sort(rng.choice(d, size=count, replace=False))


def _draw_block(w: Workload, block: int, d: int) -> np.ndarray:
    rng = np.random.default_rng([w.data_seed, block])
    n = ROW_BLOCK
    if w.dist == "normal":
        x = rng.standard_normal((n, d))
    elif w.dist == "student_t_outlier_channels":
        x = rng.standard_t(3.0, size=(n, d))
        x[:, _outlier_columns(w.data_seed, d, 8)] *= 50.0
    elif w.dist == "normal_sparse_x20":
        x = rng.standard_normal((n, d))
        mask = rng.random((n, d)) < 0.01
        x[mask] *= 20.0
    elif w.dist == "weight_outlier_columns":
        x = 0.02 * rng.standard_normal((n, d))
        x[:, _outlier_columns(w.data_seed, d, 16)] *= 30.0
    else:
        raise ValueError(w.dist)
    return x


def _rows_f64(w: Workload, row_start: int, row_count: int, d: int) -> np.ndarray:
    out = np.empty((row_count, d), dtype=np.float64)
    if row_count == 0:
        return out
    b0 = row_start // ROW_BLOCK
    b1 = (row_start + row_count - 1) // ROW_BLOCK

    def one(blk):
        x = _draw_block(w, blk, d)
        lo = max(row_start, blk * ROW_BLOCK) - blk * ROW_BLOCK
        hi = min(row_start + row_count, (blk + 1) * ROW_BLOCK) - blk * ROW_BLOCK
        pos = blk * ROW_BLOCK + lo - row_start
        out[pos:pos + (hi - lo)] = x[lo:hi]

    blocks = range(b0, b1 + 1)
    if len(blocks) > 2:
        with cf.ThreadPoolExecutor(max_workers=_threads()) as ex:
            list(ex.map(one, blocks))
    else:
        for blk in blocks:
            one(blk)
    return out


def _threads() -> int:
    try:
        return max(1, min(32, len(os.sched_getaffinity(0))))
    except AttributeError:
        return max(1, min(32, os.cpu_count() or 1))


def draw_rows(w: Workload, row_start: int = 0, row_count: Optional[int] = None,
              d: Optional[int] = None) -> np.ndarray:
    """Rows [row_start, row_start+row_count) of workload ``w`` as float64 values
    already rounded to the workload's I/O dtype (so they are exactly representable).
    """
    d = w.d if d is None else d
    if row_count is None:
        row_count = w.rows - row_start
    enc = draw_encoded(w, row_start, row_count, d)
    if w.dtype == "bf16":
        return decode_bf16(enc)
    return enc.astype(np.float64)


def draw_encoded(w: Workload, row_start: int = 0, row_count: Optional[int] = None,
                 d: Optional[int] = None) -> np.ndarray:
    """Rows [row_start, row_start+row_count) in storage form: float32, or bf16 bit
    patterns (uint16) rounded to nearest even from the float64 draws."""
    d = w.d if d is None else d
    if row_count is None:
        row_count = w.rows - row_start
    out = np.empty((row_count, d), dtype=np.uint16 if w.dtype == "bf16" else np.float32)
    step = 16 * ROW_BLOCK
    # draw and encode in slabs so float64 temporaries stay small
    for a in range(0, row_count, step):
        n = min(step, row_count - a)
        x = _rows_f64(w, row_start + a, n, d)
        if w.dtype == "bf16":
            out[a:a + n] = _encode_threads(x)
        else:
            out[a:a + n] = x.astype(np.float32)
    return out


def _encode_threads(x: np.ndarray) -> np.ndarray:
    n = x.shape[0]
    if n < 512:
        return encode_bf16(x)
    parts = np.array_split(np.arange(n), _threads())
    out = np.empty(x.shape, dtype=np.uint16)

    def one(idx):
        if idx.size:
            out[idx[0]:idx[-1] + 1] = encode_bf16(x[idx[0]:idx[-1] + 1])

    with cf.ThreadPoolExecutor(max_workers=_threads()) as ex:
        list(ex.map(one, parts))
    return out


def draw_upstream(w: Workload, row_start: int = 0, row_count: Optional[int] = None) -> np.ndarray:
    """Upstream gradients dL/dy for the calibration backward, rows [row_start,
    row_start+row_count) of i.i.d. N(0, 1) draws in the workload's storage form (float32
    or bf16 bit patterns), from a stream of their own keyed by [data seed, 0x6AD, block]."""
    if row_count is None:
        row_count = w.rows - row_start
    out = np.empty((row_count, w.d), dtype=np.uint16 if w.dtype == "bf16" else np.float32)
    first, last = row_start // ROW_BLOCK, (row_start + row_count - 1) // ROW_BLOCK if row_count else -1

    def one(blk):
        rng = np.random.default_rng([w.data_seed, 0x6AD, blk])
        x = rng.standard_normal((ROW_BLOCK, w.d))
        a, b = max(row_start, blk * ROW_BLOCK), min(row_start + row_count, (blk + 1) * ROW_BLOCK)
        part = x[a - blk * ROW_BLOCK:b - blk * ROW_BLOCK]
        out[a - row_start:b - row_start] = encode_bf16(part) if w.dtype == "bf16" else part.astype(np.float32)

    with cf.ThreadPoolExecutor(max_workers=_threads()) as ex:
        list(ex.map(one, range(first, last + 1)))
    return out


def draw_weight(w: Workload) -> np.ndarray:
    """The two-sided workload's weight matrix W (n_out x n_in), float64 values."""
    return draw_rows(w, 0, w.n_out, w.n_in)


def draw_hessian(n: int, seed: int, samples: int = 256) -> np.ndarray:
    """A seeded symmetric positive definite Hessian proxy of n x n (float64, values exact
    in float32): X^T X / samples + 0.01 I for calibration-like activations X (samples x n,
    iid N(0, 1) with 8 seeded outlier channels x20), rounded to float32 and symmetric."""
    rng = np.random.default_rng([seed, 0x4E55])
    x = rng.standard_normal((samples, n))
    x[:, np.sort(rng.choice(n, size=min(8, n), replace=False))] *= 20.0
    h = x.T @ x / samples + 0.01 * np.eye(n)
    h = 0.5 * (h + h.T)
    return h.astype(np.float32).astype(np.float64)


def sample_rows(rows: int, count: int, seed: int = 7) -> np.ndarray:
    """A seeded, sorted subset of row indices that always includes the first and
    last rows and the row just after each 256-row block boundary near them."""
    if rows <= count:
        return np.arange(rows)
    rng = np.random.default_rng([seed, rows])
    pick = set(rng.choice(rows, size=count, replace=False).tolist())
    pick.update({0, 1, rows - 1, rows - 2, min(rows - 1, ROW_BLOCK)})
    return np.array(sorted(pick), dtype=np.int64)


# ---------------------------------------------------------------------------
# rotation parameters
# ---------------------------------------------------------------------------

def draw_theta(count: int, sigma: float, seed: int) -> np.ndarray:
    """``count`` parameters iid N(0, sigma^2) (float64 values exactly representable
    in float32, since the library stores theta as float32)."""
    if sigma == 0.0:
        return np.zeros(count, dtype=np.float64)
    rng = np.random.default_rng([seed, 0x7E7A])
    return (sigma * rng.standard_normal(count)).astype(np.float32).astype(np.float64)


def quantize_theta_int8(theta: np.ndarray, stage_counts: Sequence[int]):
    """Storage encoder for int8 theta: per stage, scale = max|theta_t| / 127 (as
    float32) and q = clamp(round_half_even(theta / scale), -127, 127).

    Returns (codes int8, scales float32[m]).  The decoder (q * scale) belongs to
    the library and the oracle, each on its own.
    """
    theta = np.asarray(theta, dtype=np.float64)
    codes = np.empty(theta.shape, dtype=np.int8)
    scales = np.empty(len(stage_counts), dtype=np.float32)
    off = 0
    for t, n in enumerate(stage_counts):
        seg = theta[off:off + n]
        amax = float(np.max(np.abs(seg))) if n else 0.0
        s = np.float32(amax / 127.0) if amax > 0 else np.float32(1.0)
        scales[t] = s
        q = np.clip(np.rint(seg / np.float64(s)), -127, 127)
        codes[off:off + n] = q.astype(np.int8)
        off += n
    if off != theta.size:
        raise ValueError("stage_counts do not cover theta")
    return codes, scales

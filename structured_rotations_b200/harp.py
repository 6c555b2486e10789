"""ctypes binding of libharp (include/harp.h): argument marshalling only.

Every step of the transform runs in the library's CUDA kernels; this module
passes device pointers and the current CUDA stream through.  Loading fails
loudly when libharp.so has not been built — there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("HARP_LIB", os.path.join(_HERE, "libharp.so"))

HARP_OK = 0
HARP_ERR_INVALID_ARG = 1
HARP_ERR_SCHEDULE = 2
HARP_ERR_UNSUPPORTED = 3
HARP_ERR_NOT_MATERIALIZED = 4
HARP_ERR_ALLOC = 5
HARP_ERR_CUDA = 6
HARP_ERR_TIMEOUT = 7
HARP_ERR_WRONG_DEVICE = 8

HARP_THETA_F32 = 0
HARP_THETA_I8 = 1
HARP_F32 = 0
HARP_BF16 = 1
HARP_FORWARD = 0
HARP_INVERSE = 1

MAX_STAGES = 16

_c_i64 = ctypes.c_int64
_c_i32 = ctypes.c_int32
_c_u64 = ctypes.c_uint64
_vp = ctypes.c_void_p


class HarpError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {detail or status}")
        self.status = status


_lib = None


def lib():
    """The loaded libharp handle (raises if the library is missing)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libharp.so not found at {LIB_PATH}; build it with "
                          f"`python -m structured_rotations_b200.build`")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "harp_plan_create": (_c_i32, [ctypes.POINTER(_vp), _c_i64, ctypes.POINTER(_c_i32), _c_i32,
                                      _c_i32, _vp, ctypes.POINTER(ctypes.c_float), _c_u64, _c_u64]),
        "harp_materialize_blocks": (_c_i32, [_vp, _vp]),
        "harp_apply": (_c_i32, [_vp, _vp, _vp, _c_i64, _c_i64, _c_i64, _c_i32, _c_i32, _vp]),
        "harp_apply_ex": (_c_i32, [_vp, _vp, _vp, _c_i64, _c_i64, _c_i64, _c_i32, _c_i32, _c_i32, _vp]),
        "harp_apply_columns": (_c_i32, [_vp, _vp, _c_i64, _c_i64, _vp, _c_i64, _c_i32, _c_i32, _vp]),
        "harp_apply_host": (_c_i32, [_vp, _vp, _vp, _c_i64, _c_i64, _c_i64, _c_i32, _c_i32]),
        "harp_two_sided_workspace_bytes": (ctypes.c_size_t, [_c_i64, _c_i64]),
        "harp_apply_two_sided": (_c_i32, [_vp, _vp, _vp, _vp, _c_i64, _c_i64, _c_i64, _c_i32, _vp,
                                          ctypes.c_size_t, _vp]),
        "harp_apply_two_sided_noalloc": (_c_i32, [_vp, _vp, _vp, _vp, _c_i64, _c_i64, _c_i64, _c_i32,
                                                  _vp]),
        "harp_noalloc_scratch_bytes": (ctypes.c_size_t, []),
        "harp_plan_device_status": (_c_i32, [_vp]),
        "harp_grad_workspace_bytes": (ctypes.c_size_t, [_vp]),
        "harp_plan_compose": (_c_i32, [ctypes.POINTER(_vp), ctypes.POINTER(_vp), _c_i32, _vp]),
        "harp_apply_quant": (_c_i32, [_vp, _vp, _c_i64, _c_i64, _c_i32, _vp, _c_i64, _vp, _c_i64, _c_i32, _c_i32,
                                      _vp]),
        "harp_grad_theta": (_c_i32, [_vp, _vp, _vp, _c_i64, _c_i64, _c_i64, _c_i32, _vp, _vp, ctypes.c_size_t,
                                     _vp]),
        "harp_off_block_energy": (_c_i32, [_vp, _c_i64, _c_i64, _c_i32, _c_i32, _vp, _vp]),
        "harp_l_diag": (_c_i32, [_vp, _c_i64, _c_i64, _c_i64, _c_i32, _vp, _c_i64, _c_i32, _vp, _vp]),
        "harp_test_inject_wait_timeout": (_c_i32, [_c_i64, ctypes.c_uint32]),
        "harp_moment_check": (_c_i32, [_vp, _c_i64, _c_i64, _c_i64, _c_i32, ctypes.c_double, ctypes.c_double, _vp,
                                       _vp, _vp]),
        "harp_plan_destroy": (_c_i32, [_vp]),
        "harp_status_string": (ctypes.c_char_p, [_c_i32]),
        "harp_last_error": (ctypes.c_char_p, []),
        "harp_last_kernel": (ctypes.c_char_p, []),
        "harp_theta_count": (_c_i64, [ctypes.POINTER(_c_i32), _c_i32]),
        "harp_splitmix64": (_c_i32, [_c_u64, _c_i64, ctypes.POINTER(_c_u64)]),
        "harp_plan_base_mixer": (_c_i32, [_vp, _c_i32, ctypes.POINTER(ctypes.c_double)]),
        "harp_plan_signs": (_c_i32, [_vp, ctypes.POINTER(ctypes.c_int8)]),
        "harp_plan_shape": (_c_i32, [_vp, ctypes.POINTER(_c_i64), ctypes.POINTER(_c_i32),
                                     ctypes.POINTER(_c_i32)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _check(status: int, where: str):
    if status != HARP_OK:
        L = lib()
        detail = (L.harp_last_error() or b"").decode()
        name = L.harp_status_string(status).decode()
        raise HarpError(status, where, detail or name)


def _radices(schedule: Sequence[int]):
    arr = (_c_i32 * len(schedule))(*[int(b) for b in schedule])
    return arr


def theta_count(schedule: Sequence[int]) -> int:
    return int(lib().harp_theta_count(_radices(schedule), len(schedule)))


def splitmix64(seed: int, n: int) -> np.ndarray:
    out = np.empty(n, dtype=np.uint64)
    _check(lib().harp_splitmix64(_c_u64(seed), n, out.ctypes.data_as(ctypes.POINTER(_c_u64))),
           "harp_splitmix64")
    return out


def _stream_handle(stream) -> Optional[int]:
    if stream is None:
        import torch
        C = torch._C
        if hasattr(C, "_cuda_getCurrentRawStream"):   # the handle without a Stream object
            return C._cuda_getCurrentRawStream(C._cuda_getDevice())
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


_DTYPE = {"float32": HARP_F32, "bfloat16": HARP_BF16}


_DTYPE_OF = {}   # torch dtype -> code, filled on first use


def _dtype_code(t) -> int:
    code = _DTYPE_OF.get(t.dtype)
    if code is None:
        name = str(t.dtype).replace("torch.", "")
        if name not in _DTYPE:
            raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")
        code = _DTYPE_OF[t.dtype] = _DTYPE[name]
    return code


def _ld(t) -> int:
    if t.dim() != 2:
        raise ValueError("expected a 2-D tensor of rows")
    if t.stride(1) != 1:
        raise ValueError("rows must be contiguous (stride(1) == 1)")
    return t.stride(0) if t.shape[0] > 1 else max(t.stride(0), t.shape[1])


class Plan:
    """One HARP rotation: schedule, parameters, signs, mixers and device blocks."""

    def __init__(self, d: int, schedule: Sequence[int], theta=None, sign_seed: int = 0,
                 qr_seed: int = 0, codes=None, scales=None):
        L = lib()
        self.d = int(d)
        self.schedule = tuple(int(b) for b in schedule)
        handle = _vp()
        if codes is not None:
            codes = np.ascontiguousarray(codes, dtype=np.int8)
            scales = np.ascontiguousarray(scales, dtype=np.float32)
            kind, ptr = HARP_THETA_I8, codes.ctypes.data
            sptr = scales.ctypes.data_as(ctypes.POINTER(ctypes.c_float))
            self._keep = (codes, scales)
        else:
            kind = HARP_THETA_F32
            if theta is not None:
                theta = np.ascontiguousarray(theta, dtype=np.float32)
                ptr = theta.ctypes.data
            else:
                ptr = None
            sptr = None
            self._keep = (theta,)
        st = L.harp_plan_create(ctypes.byref(handle), self.d, _radices(self.schedule),
                                len(self.schedule), kind, ptr, sptr, _c_u64(sign_seed), _c_u64(qr_seed))
        _check(st, "harp_plan_create")
        self._h = handle

    @property
    def handle(self):
        return self._h

    @classmethod
    def compose(cls, plans: Sequence["Plan"], stream=None) -> "Plan":
        """One plan for T_{k-1} ... T_0 of materialized plans of one dimension (plans[0]
        acts first), applied in a single pass (harp_plan_compose)."""
        if not plans:
            raise ValueError("need at least one plan")
        arr = (_vp * len(plans))(*[p.handle for p in plans])
        handle = _vp()
        _check(lib().harp_plan_compose(ctypes.byref(handle), arr, len(plans), _stream_handle(stream)),
               "harp_plan_compose")
        c = cls.__new__(cls)
        c.d = plans[0].d
        c.schedule = tuple(b for p in plans for b in p.schedule)
        c._keep = ()
        c._h = handle
        c.composite = True
        return c

    def materialize(self, stream=None) -> "Plan":
        _check(lib().harp_materialize_blocks(self._h, _stream_handle(stream)), "harp_materialize_blocks")
        return self

    def apply(self, x, y=None, direction: str = "forward", stream=None, rows: Optional[int] = None):
        """y = T x (forward) or T^T x (inverse) row by row; y defaults to a new tensor."""
        import torch
        if y is None:
            y = torch.empty_like(x)
        if x.dtype != y.dtype:
            raise TypeError("x and y must share a dtype")
        if x.shape[-1] != self.d or y.shape[-1] != self.d:
            raise ValueError(f"last dimension must be d={self.d}")
        n = x.shape[0] if rows is None else rows
        d = HARP_FORWARD if direction == "forward" else HARP_INVERSE
        _check(lib().harp_apply(self._h, x.data_ptr(), y.data_ptr(), n, _ld(x), _ld(y),
                                _dtype_code(x), d, _stream_handle(stream)), "harp_apply")
        return y

    def apply_quant(self, x, qblock: int = 128, direction: str = "forward", q=None, scales=None, stream=None):
        """T x (or T^T x) with the fused blockwise quantizer (harp_apply_quant): bf16 rows in,
        int8 codes [rows, d] and float32 scales [rows, d / qblock] out, y ~= q * scale per
        aligned block of qblock coordinates.  Returns (q, scales)."""
        import torch
        if x.shape[-1] != self.d:
            raise ValueError(f"last dimension must be d={self.d}")
        rows = x.shape[0]
        if q is None:
            q = torch.empty(rows, self.d, dtype=torch.int8, device=x.device)
        if scales is None:
            scales = torch.empty(rows, max(1, self.d // qblock), dtype=torch.float32, device=x.device)
        d = HARP_FORWARD if direction == "forward" else HARP_INVERSE
        _check(lib().harp_apply_quant(self._h, x.data_ptr(), rows, _ld(x), _dtype_code(x), q.data_ptr(), _ld(q),
                                      scales.data_ptr(), _ld(scales), qblock, d, _stream_handle(stream)),
               "harp_apply_quant")
        return q, scales

    def grad_theta(self, x, g, dtheta=None, workspace=None, stream=None):
        """dL/dtheta for L = sum_r g_r . (T x_r) (harp_grad_theta): the calibration backward
        through the forward transform, for rows x and upstream gradients g = dL/dy of one
        dtype on the GPU.  Returns a float32 tensor of theta_count entries (dtheta, if
        given, is filled).  dL/dx is self.apply(g, direction="inverse")."""
        import torch
        if x.dtype != g.dtype or x.shape != g.shape or x.shape[-1] != self.d:
            raise ValueError(f"x and g must be rows of d={self.d} of one dtype")
        # a composite's schedule is its plans' schedules in a row (no theta count of its
        # own): the library declines it, so any buffer does
        n = theta_count(self.schedule) if not getattr(self, "composite", False) else 1
        if dtheta is None:
            dtheta = torch.empty(n, dtype=torch.float32, device=x.device)
        if dtheta.dtype != torch.float32 or dtheta.numel() != n or not dtheta.is_contiguous():
            raise ValueError(f"dtheta must be a contiguous float32 tensor of {n} entries")
        need = int(lib().harp_grad_workspace_bytes(self._h))
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
        _check(lib().harp_grad_theta(self._h, x.data_ptr(), g.data_ptr(), x.shape[0], _ld(x), _ld(g),
                                     _dtype_code(x), dtheta.data_ptr(), workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(), _stream_handle(stream)),
               "harp_grad_theta")
        return dtheta

    def apply_host(self, x, y=None, direction: str = "forward"):
        """Rows of a host (CPU) tensor through the GPU and back (harp_apply_host): copies,
        kernels and copies overlap in chunks; pin x and y (tensor.pin_memory()) for the
        overlap.  Returns y (a new host tensor by default)."""
        import torch
        if x.device.type != "cpu":
            raise ValueError("apply_host takes host tensors; use apply for device tensors")
        if y is None:
            y = torch.empty_like(x, pin_memory=x.is_pinned())
        if x.dtype != y.dtype or x.shape != y.shape or x.shape[-1] != self.d:
            raise ValueError(f"x and y must be rows of d={self.d} of one dtype")
        d = HARP_FORWARD if direction == "forward" else HARP_INVERSE
        _check(lib().harp_apply_host(self._h, x.data_ptr(), y.data_ptr(), x.shape[0], _ld(x), _ld(y),
                                     _dtype_code(x), d), "harp_apply_host")
        return y

    def apply_ex(self, x, y, direction: str = "forward", stream=None):
        """Rows of x (float32 or bfloat16) into y of its own type (harp_apply_ex), e.g. bf16
        rows into an fp32 intermediate."""
        if x.shape[-1] != self.d or y.shape[-1] != self.d or x.shape[0] != y.shape[0]:
            raise ValueError(f"x and y must both be rows of d={self.d}")
        d = HARP_FORWARD if direction == "forward" else HARP_INVERSE
        _check(lib().harp_apply_ex(self._h, x.data_ptr(), y.data_ptr(), x.shape[0], _ld(x), _ld(y),
                                   _dtype_code(x), _dtype_code(y), d, _stream_handle(stream)), "harp_apply_ex")
        return y

    def apply_columns(self, x, y=None, direction: str = "forward", stream=None):
        """Every column of the fp32 matrix x (d rows) takes T or T^T (harp_apply_columns);
        y defaults to x itself (in place); a bfloat16 y receives the rounded result.  x is
        overwritten either way."""
        import torch
        if x.dtype != torch.float32 or x.shape[0] != self.d:
            raise ValueError(f"x must be float32 with d={self.d} rows")
        if y is None:
            y = x
        if y.shape != x.shape:
            raise ValueError("y must have the shape of x")
        d = HARP_FORWARD if direction == "forward" else HARP_INVERSE
        _check(lib().harp_apply_columns(self._h, x.data_ptr(), _ld(x), x.shape[1], y.data_ptr(), _ld(y),
                                        _dtype_code(y), d, _stream_handle(stream)), "harp_apply_columns")
        return y

    def device_status(self) -> None:
        """Synchronize and raise HarpError(HARP_ERR_TIMEOUT) if a bounded device
        wait of a kernel launched with this plan gave up."""
        _check(lib().harp_plan_device_status(self._h), "harp_plan_device_status")

    def base_mixer(self, radix: int) -> np.ndarray:
        out = np.empty((radix, radix), dtype=np.float64)
        _check(lib().harp_plan_base_mixer(self._h, radix, out.ctypes.data_as(ctypes.POINTER(ctypes.c_double))),
               "harp_plan_base_mixer")
        return out

    def signs(self) -> np.ndarray:
        out = np.empty(self.d, dtype=np.int8)
        _check(lib().harp_plan_signs(self._h, out.ctypes.data_as(ctypes.POINTER(ctypes.c_int8))),
               "harp_plan_signs")
        return out

    def shape(self):
        d = _c_i64()
        m = _c_i32()
        r = (_c_i32 * MAX_STAGES)()
        _check(lib().harp_plan_shape(self._h, ctypes.byref(d), ctypes.byref(m), r), "harp_plan_shape")
        return d.value, tuple(r[: m.value])

    def close(self):
        if getattr(self, "_h", None):
            lib().harp_plan_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def last_kernel() -> str:
    """Name of the last kernel launched by this thread through the library."""
    return (lib().harp_last_kernel() or b"").decode()


def workspace_bytes(n_out: int, n_in: int) -> int:
    return int(lib().harp_two_sided_workspace_bytes(n_out, n_in))


def apply_two_sided(plan_u: Plan, plan_v: Plan, w, w_out=None, workspace=None, stream=None):
    """W_out = T_U^T W T_V (U on the output side, V on the input side)."""
    import torch
    n_out, n_in = w.shape
    if w_out is None:
        w_out = torch.empty_like(w)
    need = workspace_bytes(n_out, n_in)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=w.device)
    ld = _ld(w)
    if _ld(w_out) != ld:
        raise ValueError("W and W_out must share a leading dimension")
    _check(lib().harp_apply_two_sided(plan_u.handle, plan_v.handle, w.data_ptr(), w_out.data_ptr(),
                                      n_out, n_in, ld, _dtype_code(w), workspace.data_ptr(),
                                      workspace.numel() * workspace.element_size(),
                                      _stream_handle(stream)), "harp_apply_two_sided")
    return w_out


def off_block_energy(h, q: int, out=None, stream=None):
    """(energy of the square matrix h outside its q x q diagonal blocks, total energy) as a
    device float64 tensor of 2 (harp_off_block_energy); R_bd = out[0] / out[1]."""
    import torch
    n = h.shape[0]
    if h.dim() != 2 or h.shape[1] != n:
        raise ValueError("h must be square")
    if out is None:
        out = torch.empty(2, dtype=torch.float64, device=h.device)
    _check(lib().harp_off_block_energy(h.data_ptr(), n, _ld(h), _dtype_code(h), q, out.data_ptr(),
                                       _stream_handle(stream)), "harp_off_block_energy")
    return out


def l_diag(w, h, qblock: int, out=None, stream=None):
    """sum_j h_jj sum_r (w_rj - Q(w)_rj)^2 with Q the blockwise int8 quantizer along the rows
    (harp_l_diag), as a device float64 tensor of 1; h is float32 (only its diagonal is read)."""
    import torch
    rows, cols = w.shape
    if h.dtype != torch.float32 or h.shape[0] < cols or h.shape[1] < cols:
        raise ValueError("h must be a float32 matrix of at least cols x cols")
    if out is None:
        out = torch.empty(1, dtype=torch.float64, device=w.device)
    _check(lib().harp_l_diag(w.data_ptr(), rows, cols, _ld(w), _dtype_code(w), h.data_ptr(), _ld(h), qblock,
                             out.data_ptr(), _stream_handle(stream)), "harp_l_diag")
    return out


def inject_wait_timeout(poll_limit: int = 0, extra_bytes: int = 0) -> None:
    """Test hook (harp_test_inject_wait_timeout): make the staging waits of this thread's
    next tiled-kernel launches run out after poll_limit polls; (0, 0) clears it."""
    _check(lib().harp_test_inject_wait_timeout(poll_limit, extra_bytes), "harp_test_inject_wait_timeout")


def moment_check(x, tau1: float = 0.0, tau2: float = 0.0, moments=None, passes=None, stream=None):
    """Per row of the device rows x (harp_moment_check): (sum x^2, sum |x|^3, sum x^4) as a float64
    tensor [rows, 3], and the number of composed passes (1 if m4 / m2^2 <= tau1, 2 if <= tau2, else
    3) as an int32 tensor [rows].  Returns (moments, passes)."""
    import torch
    rows, d = x.shape
    if moments is None:
        moments = torch.empty(rows, 3, dtype=torch.float64, device=x.device)
    if passes is None:
        passes = torch.empty(rows, dtype=torch.int32, device=x.device)
    _check(lib().harp_moment_check(x.data_ptr(), rows, d, _ld(x), _dtype_code(x), float(tau1), float(tau2),
                                   moments.data_ptr(), passes.data_ptr(), _stream_handle(stream)),
           "harp_moment_check")
    return moments, passes

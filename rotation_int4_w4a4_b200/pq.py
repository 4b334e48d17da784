"""ctypes binding for libpq (``include/pq.h``): the same entry points, argument marshalling only.

Tensors are passed as device pointers (``torch.Tensor.data_ptr()``) with the current CUDA
stream unless one is given.  Every call checks the returned status and raises ``PQError``
with the library's message.  Importing this module loads the library and raises if it has
not been built (``python -m rotation_int4_w4a4_b200.build``): there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "_lib", "libpq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libpq.so is not built ({_LIB_PATH}); run python -m rotation_int4_w4a4_b200.build")
lib = ctypes.CDLL(_LIB_PATH)

PQ_OK, PQ_ERR_INVALID_ARG, PQ_ERR_UNSUPPORTED, PQ_ERR_CUDA, PQ_ERR_ALLOC, PQ_ERR_TIMEOUT = range(6)
PQ_HADAMARD, PQ_GIVENS, PQ_SMOOTH_HADAMARD = range(3)
PQ_OUT_F32, PQ_OUT_BF16 = range(2)
PQ_FLAG_SMOOTH_AFTER_ROTATE = 0x1
PQ_NO_PAIR = 0xFF
KINDS = {"hadamard": PQ_HADAMARD, "givens": PQ_GIVENS, "smooth_hadamard": PQ_SMOOTH_HADAMARD}

# Every symbol the header declares.
EXPORTS = ("pq_select_pairs", "pq_make_plan", "pq_destroy_plan", "pq_transform_quant",
           "pq_pack_weights", "pq_w4a4_gemm", "pq_w4a4_gemm_noalloc", "pq_w4a4_gemm_launch_count",
           "pq_w4a4_gemm_launch_count_g", "pq_w4a4_linear", "pq_make_plan_outliers",
           "pq_rrs_prepare", "pq_rrs_transform_quant", "pq_rrs_pack_weights", "pq_rrs_gemm",
           "pq_check_status",
           "pq_selftest_wait_timeout", "pq_status_string", "pq_last_error")

_c = ctypes
_vp, _i64, _u64, _i32, _u32 = _c.c_void_p, _c.c_int64, _c.c_uint64, _c.c_int, _c.c_uint32
lib.pq_select_pairs.argtypes = [_u64, _i32, _i32, _i32, _i32, _vp]
lib.pq_select_pairs.restype = _i32
lib.pq_make_plan.argtypes = [_c.POINTER(_vp), _i32, _i32, _i32, _i32, _vp, _vp, _vp, _u32]
lib.pq_make_plan.restype = _i32
lib.pq_make_plan_outliers.argtypes = [_c.POINTER(_vp), _i32, _i32, _i32, _i32, _vp, _vp, _vp, _u32, _i32, _vp]
lib.pq_make_plan_outliers.restype = _i32
lib.pq_destroy_plan.argtypes = [_vp]
lib.pq_destroy_plan.restype = None
lib.pq_transform_quant.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp]
lib.pq_transform_quant.restype = _i32
lib.pq_pack_weights.argtypes = [_vp, _vp, _i64, _vp, _vp, _vp, _vp]
lib.pq_pack_weights.restype = _i32
lib.pq_w4a4_gemm.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _vp, _i32, _vp]
lib.pq_w4a4_gemm.restype = _i32
lib.pq_w4a4_gemm_noalloc.argtypes = lib.pq_w4a4_gemm.argtypes
lib.pq_w4a4_gemm_noalloc.restype = _i32
lib.pq_w4a4_gemm_launch_count.argtypes = [_i64, _i64, _i64, _c.POINTER(_i32)]
lib.pq_w4a4_gemm_launch_count.restype = _i32
lib.pq_w4a4_gemm_launch_count_g.argtypes = [_i64, _i64, _i64, _i32, _c.POINTER(_i32)]
lib.pq_w4a4_gemm_launch_count_g.restype = _i32
lib.pq_w4a4_linear.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i64, _vp, _i32, _vp]
lib.pq_w4a4_linear.restype = _i32
lib.pq_rrs_prepare.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp]
lib.pq_rrs_prepare.restype = _i32
lib.pq_rrs_transform_quant.argtypes = [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp]
lib.pq_rrs_transform_quant.restype = _i32
lib.pq_rrs_pack_weights.argtypes = [_vp, _vp, _i64, _vp, _vp, _vp, _vp, _vp]
lib.pq_rrs_pack_weights.restype = _i32
lib.pq_rrs_gemm.argtypes = [_vp, _vp, _vp, _vp, _i64, _i64, _i64, _i32, _vp, _i32, _vp]
lib.pq_rrs_gemm.restype = _i32
lib.pq_selftest_wait_timeout.argtypes = [_u64, _vp]
lib.pq_selftest_wait_timeout.restype = _i32
lib.pq_check_status.argtypes = [_vp, _vp]
lib.pq_check_status.restype = _i32
lib.pq_status_string.argtypes = [_i32]
lib.pq_status_string.restype = _c.c_char_p
lib.pq_last_error.argtypes = []
lib.pq_last_error.restype = _c.c_char_p


class PQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.pq_last_error().decode(errors="replace")
        super().__init__(f"{where}: {lib.pq_status_string(status).decode()}: {msg}")


def _check(status: int, where: str) -> None:
    if status != PQ_OK:
        raise PQError(status, where)


def _ptr(x, rows_strided=False):
    """Device pointer of a tensor (None -> NULL; an int passes through as a raw address).

    The library reads and writes dense row-major device buffers, so a tensor must live on a
    CUDA device and be contiguous; with rows_strided (the activations, whose row stride is
    passed as ldx) only the last dimension must be contiguous.  Anything else would be read at
    the wrong addresses, so it is rejected here instead.
    """
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not getattr(x, "is_cuda", False):
        raise ValueError("expected a CUDA tensor: the library takes device pointers")
    if not (x.stride(-1) == 1 if rows_strided else x.is_contiguous()):
        raise ValueError("expected a contiguous tensor" + (" along its last dimension" if rows_strided else ""))
    return x.data_ptr()


def _arg(x, name, dtype, need, rows_strided=False):
    """Pointer of a tensor argument after checking its dtype and that it holds at least `need`
    elements (the C ABI only sees a pointer: a wrong dtype or a short buffer would make the
    kernels read or write past its end).  Raw integer addresses pass unchecked."""
    if x is None or isinstance(x, int):
        return _ptr(x)
    import torch
    want = {"bf16": (torch.bfloat16,), "u8": (torch.uint8,), "f32": (torch.float32,),
            "i32": (torch.int32,), "y": (torch.float32, torch.bfloat16)}[dtype]
    if x.dtype not in want:
        raise ValueError(f"{name}: dtype {x.dtype} is not accepted (expected {' or '.join(map(str, want))})")
    p = _ptr(x, rows_strided)
    if rows_strided:
        if x.dim() != 2:
            raise ValueError(f"{name}: expected a 2-D tensor")
        extent = (x.shape[0] - 1) * x.stride(0) + x.shape[1] if x.shape[0] > 0 else 0
    else:
        extent = x.numel()
    if extent < need:
        raise ValueError(f"{name}: holds {extent} elements, the call needs {need}")
    return p


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def pq_select_pairs(seed: int, D: int, g: int, K: int, N: int) -> np.ndarray:
    """Host-side greedy pair selection -> uint8 [D/g, K, g/2, 2] (0xFF = no pair)."""
    out = np.empty((D // g, K, g // 2, 2), dtype=np.uint8)
    _check(lib.pq_select_pairs(seed, D, g, K, N, out.ctypes.data), "pq_select_pairs")
    return out


class Plan:
    """Owns a ``pq_plan`` (device tables); freed by :meth:`close` or garbage collection."""

    def __init__(self, kind, D: int, g: int = 128, K: int = 0, pairs=None, angles=None,
                 beta=None, flags: int = 0, groups8=None):
        """groups8: group indices kept as 8-bit outlier groups (codes and scales then hold
        Gx = D/g + 3 len(groups8) groups per row; see ``Dx``)."""
        kind = KINDS.get(kind, kind)
        self.kind, self.D, self.g, self.K, self.flags = kind, D, g, K, flags
        self.groups8 = [] if groups8 is None else [int(v) for v in groups8]
        self.Gx = D // g + 3 * len(self.groups8)
        self.Dx = self.Gx * g            # the GEMM's reduction length for this plan's codes
        keep = []

        def host(a, dt):
            if a is None:
                return None
            a = np.ascontiguousarray(a, dtype=dt)
            keep.append(a)
            return a.ctypes.data

        h = _vp()
        if self.groups8:
            _check(lib.pq_make_plan_outliers(_c.byref(h), kind, D, g, K, host(pairs, np.uint8),
                                             host(angles, np.float32), host(beta, np.float32), flags,
                                             len(self.groups8), host(self.groups8, np.int32)),
                   "pq_make_plan_outliers")
        else:
            _check(lib.pq_make_plan(_c.byref(h), kind, D, g, K, host(pairs, np.uint8),
                                    host(angles, np.float32), host(beta, np.float32), flags),
                   "pq_make_plan")
        self._h = h

    @property
    def handle(self):
        return self._h

    def close(self):
        if getattr(self, "_h", None):
            lib.pq_destroy_plan(self._h)
            self._h = None

    def __del__(self):  # pragma: no cover - interpreter teardown order
        try:
            self.close()
        except Exception:
            pass


def pq_make_plan(kind, D, g=128, K=0, pairs=None, angles=None, beta=None, flags=0) -> Plan:
    return Plan(kind, D, g, K, pairs, angles, beta, flags)


def pq_destroy_plan(plan: Plan) -> None:
    plan.close()


def pq_transform_quant(plan: Plan, X, codes, scales, smooth_out=None, T=None, ldx=None,
                       stream=None) -> None:
    """X bf16 [T, ldx] -> codes uint8 [T, Dx/2], scales float32 [T, Gx] (device tensors;
    Dx = D and Gx = D/g unless the plan has 8-bit groups)."""
    T = X.shape[0] if T is None else T
    ldx = X.stride(0) if ldx is None else ldx
    D, G = plan.D, plan.Gx
    if not isinstance(X, int) and X.dim() == 2 and X.stride(0) != ldx:
        raise ValueError(f"X: row stride {X.stride(0)} differs from ldx={ldx}")
    xp = _arg(X, "X", "bf16", (T - 1) * ldx + D if T > 0 else 0, rows_strided=True)
    _check(lib.pq_transform_quant(plan.handle, xp, T, ldx, _arg(codes, "codes", "u8", T * plan.Dx // 2),
                                  _arg(scales, "scales", "f32", T * G),
                                  _arg(smooth_out, "smooth_out", "f32", -(-T // 128) * D),
                                  _stream(stream)), "pq_transform_quant")


def pq_pack_weights(plan: Plan, W, codes_W, scales_W, smooth_w=None, N=None, stream=None) -> None:
    """W bf16 [N, D] -> codes_W uint8 [N, Dx/2], scales_W float32 [N, Gx] (device tensors)."""
    N = W.shape[0] if N is None else N
    D, G = plan.D, plan.Gx
    _check(lib.pq_pack_weights(plan.handle, _arg(W, "W", "bf16", N * D), N,
                               _arg(smooth_w, "smooth_w", "f32", D),
                               _arg(codes_W, "codes_W", "u8", N * plan.Dx // 2),
                               _arg(scales_W, "scales_W", "f32", N * G), _stream(stream)),
           "pq_pack_weights")


def pq_w4a4_gemm(codes_A, scales_A, codes_W, scales_W, Y, T=None, N=None, D=None, g=128,
                 out_dtype=None, stream=None) -> None:
    """Y [T, N] = per-group scaled int4 x int4 product (device tensors)."""
    T, N, D, out_dtype, ptrs = _gemm_args(codes_A, scales_A, codes_W, scales_W, Y, T, N, D, g, out_dtype)
    _check(lib.pq_w4a4_gemm(*ptrs[:4], T, N, D, g, ptrs[4], out_dtype, _stream(stream)), "pq_w4a4_gemm")


def _gemm_args(codes_A, scales_A, codes_W, scales_W, Y, T, N, D, g, out_dtype, sa_per_token=False):
    """Sizes, output dtype and checked pointers shared by the two GEMM entry points."""
    T = codes_A.shape[0] if T is None else T
    N = codes_W.shape[0] if N is None else N
    D = codes_A.shape[1] * 2 if D is None else D
    if not isinstance(Y, int):
        import torch
        y_kind = PQ_OUT_BF16 if Y.dtype == torch.bfloat16 else PQ_OUT_F32
        if out_dtype is None:
            out_dtype = y_kind
        elif out_dtype != y_kind or Y.dtype not in (torch.float32, torch.bfloat16):
            raise ValueError(f"Y: dtype {Y.dtype} does not match out_dtype={out_dtype}")
    elif out_dtype is None:
        out_dtype = PQ_OUT_F32
    G = D // g if g else 0
    ptrs = (_arg(codes_A, "codes_A", "u8", T * D // 2),
            _arg(scales_A, "token_scales" if sa_per_token else "scales_A", "f32", T if sa_per_token else T * G),
            _arg(codes_W, "codes_W", "u8", N * D // 2), _arg(scales_W, "scales_W", "f32", N * G),
            _arg(Y, "Y", "y", T * N))
    return T, N, D, out_dtype, ptrs


def pq_w4a4_gemm_noalloc(codes_A, scales_A, codes_W, scales_W, Y, T=None, N=None, D=None, g=128,
                         out_dtype=None, stream=None) -> None:
    """:func:`pq_w4a4_gemm` with the library's fixed scratch; (T + N) * D <= NOALLOC_SCRATCH_BYTES."""
    T, N, D, out_dtype, ptrs = _gemm_args(codes_A, scales_A, codes_W, scales_W, Y, T, N, D, g, out_dtype)
    _check(lib.pq_w4a4_gemm_noalloc(*ptrs[:4], T, N, D, g, ptrs[4], out_dtype, _stream(stream)),
           "pq_w4a4_gemm_noalloc")


def pq_w4a4_linear(plan: Plan, X, codes_A, scales_A, codes_W, scales_W, Y, T=None, ldx=None, N=None,
                   out_dtype=None, stream=None) -> None:
    """Transform X into codes_A / scales_A and multiply with the packed weights into Y, one call
    (for T <= 128 the GEMM overlaps the transform as its programmatic dependent)."""
    T = X.shape[0] if T is None else T
    ldx = X.stride(0) if ldx is None else ldx
    N = codes_W.shape[0] if N is None else N
    D, g = plan.D, plan.g
    xp = _arg(X, "X", "bf16", (T - 1) * ldx + D if T > 0 else 0, rows_strided=True)
    T, N, _, out_dtype, ptrs = _gemm_args(codes_A, scales_A, codes_W, scales_W, Y, T, N, plan.Dx, g, out_dtype)
    _check(lib.pq_w4a4_linear(plan.handle, xp, T, ldx, ptrs[0], ptrs[1], ptrs[2], ptrs[3], N, ptrs[4], out_dtype,
                              _stream(stream)), "pq_w4a4_linear")


def pq_rrs_prepare(plan: Plan, X, chan_max, perm, inv_perm, group_scale, T=None, ldx=None, stream=None) -> None:
    """Channel maxima of the rotated activations, their descending order and the smoothing scale
    of each reordered group of 128 (device tensors: float32 [D], int32 [D], int32 [D], float32 [G])."""
    T = X.shape[0] if T is None else T
    ldx = X.stride(0) if ldx is None else ldx
    D, G = plan.D, plan.D // plan.g
    xp = _arg(X, "X", "bf16", (T - 1) * ldx + D if T > 0 else 0, rows_strided=True)
    _check(lib.pq_rrs_prepare(plan.handle, xp, T, ldx, _arg(chan_max, "chan_max", "f32", D),
                              _arg(perm, "perm", "i32", D), _arg(inv_perm, "inv_perm", "i32", D),
                              _arg(group_scale, "group_scale", "f32", G), _stream(stream)), "pq_rrs_prepare")


def pq_rrs_transform_quant(plan: Plan, X, perm, group_scale, codes, token_scales, T=None, ldx=None,
                           stream=None) -> None:
    """Smoothed, reordered activations quantised per token: codes uint8 [T, D/2], float32 [T]."""
    T = X.shape[0] if T is None else T
    ldx = X.stride(0) if ldx is None else ldx
    D, G = plan.D, plan.D // plan.g
    xp = _arg(X, "X", "bf16", (T - 1) * ldx + D if T > 0 else 0, rows_strided=True)
    _check(lib.pq_rrs_transform_quant(plan.handle, xp, T, ldx, _arg(perm, "perm", "i32", D),
                                      _arg(group_scale, "group_scale", "f32", G),
                                      _arg(codes, "codes", "u8", T * D // 2),
                                      _arg(token_scales, "token_scales", "f32", T), _stream(stream)),
           "pq_rrs_transform_quant")


def pq_rrs_pack_weights(plan: Plan, W, perm, group_scale, codes_W, scales_W, N=None, stream=None) -> None:
    """Reordered weights quantised per group, smoothing scales folded into scales_W [N, G]."""
    N = W.shape[0] if N is None else N
    D, G = plan.D, plan.D // plan.g
    _check(lib.pq_rrs_pack_weights(plan.handle, _arg(W, "W", "bf16", N * D), N, _arg(perm, "perm", "i32", D),
                                   _arg(group_scale, "group_scale", "f32", G),
                                   _arg(codes_W, "codes_W", "u8", N * D // 2),
                                   _arg(scales_W, "scales_W", "f32", N * G), _stream(stream)),
           "pq_rrs_pack_weights")


def pq_rrs_gemm(codes_A, token_scales, codes_W, scales_W, Y, T=None, N=None, D=None, g=128, out_dtype=None,
                stream=None) -> None:
    """Y [T, N] = token_scales[t] * sum_G scales_W[n, G] d_G (device tensors)."""
    T = codes_A.shape[0] if T is None else T
    N = codes_W.shape[0] if N is None else N
    D = codes_A.shape[1] * 2 if D is None else D
    T, N, D, out_dtype, ptrs = _gemm_args(codes_A, token_scales, codes_W, scales_W, Y, T, N, D, g, out_dtype,
                                          sa_per_token=True)
    _check(lib.pq_rrs_gemm(*ptrs[:4], T, N, D, g, ptrs[4], out_dtype, _stream(stream)), "pq_rrs_gemm")


def pq_w4a4_gemm_launch_count_g(T: int, N: int, D: int, g: int) -> int:
    """Kernels one pq_w4a4_gemm call of these sizes and group size launches on the current device."""
    n = _i32(0)
    _check(lib.pq_w4a4_gemm_launch_count_g(T, N, D, g, _c.byref(n)), "pq_w4a4_gemm_launch_count_g")
    return n.value


def pq_w4a4_gemm_launch_count(T: int, N: int, D: int) -> int:
    """Kernels one pq_w4a4_gemm call of these sizes launches on the current device (2 or 3)."""
    n = _i32(0)
    _check(lib.pq_w4a4_gemm_launch_count(T, N, D, _c.byref(n)), "pq_w4a4_gemm_launch_count")
    return n.value


def pq_selftest_wait_timeout(limit_ns: int, stream=None) -> None:
    """Launch the bounded-wait diagnostic; the next pq_check_status reports PQ_ERR_TIMEOUT."""
    _check(lib.pq_selftest_wait_timeout(limit_ns, _stream(stream)), "pq_selftest_wait_timeout")


def pq_check_status(plan: Plan | None = None, stream=None) -> int:
    """Synchronise and return the status code (raises PQError on failure)."""
    st = lib.pq_check_status(plan.handle if plan is not None else None, _stream(stream))
    _check(st, "pq_check_status")
    return st

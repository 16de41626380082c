"""SmoothQuant W8A8 INT8 linear layer for NVIDIA B200 (sm_100a).

Thin Python binding over libsq (the C ABI in include/sq.h).  Every function
here only marshals arguments -- tensors become device pointers, the current
torch CUDA stream becomes the stream argument -- and raises ``SQError`` when
the library returns an error.  All arithmetic runs in the library's CUDA
kernels; there is no CPU fallback: if libsq.so cannot be loaded, every call
raises.

The raw entry points keep the C names and take caller-allocated outputs:

    sq_calib_absmax(x, ax)                      ax[K] accumulated by max
    sq_smooth_factors(ax, w, alpha, s, aw=None)
    sq_smooth_quant_weight(w, s, wq, sw)
    sq_quant_act(x, s, xq, sx)
    sq_w8a8_gemm(xq, sx, wq, sw, y)
    sq_w8a8_gemm_ws(xq, sx, wq, sw, y, workspace)   every SM busy whatever the shape
    sq_w8a8_gemm_workspace_size(M, N, K)
    sq_w8a8_gemm_s32(xq, wq, acc)
    sq_linear(x, s, wq, sw, y, workspace)
    sq_linear_workspace_size(M, N, K)
    sq_linear_noalloc(x, s, wq, sw, y)          no workspace, no allocation
    sq_device_status()

``calibrate``, ``prepare_weight`` and ``linear`` are conveniences that allocate
their outputs with torch and call the raw entry points.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional, Tuple

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsq.so")

SQ_OK, SQ_ERR_INVALID_ARG, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA, SQ_ERR_TIMEOUT = range(5)
SQ_F32, SQ_BF16 = 0, 1

# every symbol include/sq.h declares
ABI_SYMBOLS = (
    "sq_status_string",
    "sq_version",
    "sq_calib_absmax",
    "sq_smooth_factors",
    "sq_smooth_quant_weight",
    "sq_quant_act",
    "sq_fold_gamma",
    "sq_rmsnorm_quant",
    "sq_silu_mul_quant",
    "sq_gptq_workspace_size",
    "sq_gptq_hessian",
    "sq_gptq_factor",
    "sq_gptq_quant_weight",
    "sq_w8a8_gemm",
    "sq_w8a8_gemm_ws",
    "sq_w8a8_gemm_workspace_size",
    "sq_w8a8_gemm_s32",
    "sq_linear",
    "sq_linear_workspace_size",
    "sq_linear_noalloc",
    "sq_device_status",
    "sq_selftest_wait_timeout",
)


class SQError(RuntimeError):
    def __init__(self, fn: str, status: int, name: str):
        super().__init__(f"{fn} failed: {name} ({status})")
        self.status = status
        self.fn = fn


_lock = threading.Lock()
_lib = None


def _declare(lib):
    P, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float
    E = ctypes.c_int
    sig = {
        "sq_status_string": ([E], ctypes.c_char_p),
        "sq_version": ([], ctypes.c_int),
        "sq_calib_absmax": ([P, E, I, I, I, P, P], E),
        "sq_smooth_factors": ([P, P, E, I, I, F, P, P, P], E),
        "sq_smooth_quant_weight": ([P, E, I, I, P, P, P, P], E),
        "sq_quant_act": ([P, E, I, I, P, P, P, P], E),
        "sq_fold_gamma": ([P, P, I, P, P], E),
        "sq_rmsnorm_quant": ([P, E, I, I, P, F, P, P, P, P], E),
        "sq_silu_mul_quant": ([P, E, I, I, P, P, P, P, P], E),
        "sq_gptq_workspace_size": ([I], ctypes.c_size_t),
        "sq_gptq_hessian": ([P, E, I, I, P, P, P], E),
        "sq_gptq_factor": ([P, I, F, P, P, ctypes.c_size_t, P], E),
        "sq_gptq_quant_weight": ([P, E, I, I, P, P, P, P, P], E),
        "sq_w8a8_gemm": ([P, P, P, P, I, I, I, P, E, P], E),
        "sq_w8a8_gemm_ws": ([P, P, P, P, I, I, I, P, E, P, ctypes.c_size_t, P], E),
        "sq_w8a8_gemm_workspace_size": ([I, I, I], ctypes.c_size_t),
        "sq_w8a8_gemm_s32": ([P, P, I, I, I, P, P], E),
        "sq_linear": ([P, E, P, P, P, I, I, I, P, E, P, ctypes.c_size_t, P], E),
        "sq_linear_workspace_size": ([I, I, I], ctypes.c_size_t),
        "sq_linear_noalloc": ([P, E, P, P, P, I, I, I, P, E, P], E),
        "sq_device_status": ([P, ctypes.POINTER(ctypes.c_uint32)], E),
        "sq_selftest_wait_timeout": ([ctypes.c_uint32, P], E),
    }
    for name, (args, res) in sig.items():
        f = getattr(lib, name)
        f.argtypes = args
        f.restype = res


def lib():
    """The loaded libsq (ctypes.CDLL).  Raises if the library is not built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(
                    f"libsq.so is not built at {LIB_PATH}; run "
                    "`python -m w8a8_int8_gemm_channel_b200._build` (needs nvcc)"
                )
            l = ctypes.CDLL(LIB_PATH)
            _declare(l)
            _lib = l
    return _lib


def status_string(st: int) -> str:
    return lib().sq_status_string(st).decode()


def _check(fn: str, st: int):
    if st != SQ_OK:
        raise SQError(fn, st, status_string(st))


def _torch():
    import torch

    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return SQ_F32
    if t.dtype == torch.bfloat16:
        return SQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; expected float32 or bfloat16")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("libsq takes device tensors")
    if not t.is_contiguous():
        raise ValueError("libsq takes contiguous tensors")
    return t.data_ptr()


def _stream(stream=None) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


# ---------------------------------------------------------------------------
# raw entry points (C names)
# ---------------------------------------------------------------------------

def sq_calib_absmax(x, ax, stream=None):
    T, K = x.shape
    _check("sq_calib_absmax",
           lib().sq_calib_absmax(_ptr(x), _dtype_code(x), T, K, K, _ptr(ax), _stream(stream)))


def sq_smooth_factors(ax, w, alpha: float, s, aw=None, stream=None):
    N, K = w.shape
    _check("sq_smooth_factors",
           lib().sq_smooth_factors(_ptr(ax), _ptr(w), _dtype_code(w), N, K, float(alpha), _ptr(s),
                                   _ptr(aw), _stream(stream)))


def sq_smooth_quant_weight(w, s, wq, sw, stream=None):
    N, K = w.shape
    _check("sq_smooth_quant_weight",
           lib().sq_smooth_quant_weight(_ptr(w), _dtype_code(w), N, K, _ptr(s), _ptr(wq), _ptr(sw),
                                        _stream(stream)))


def sq_quant_act(x, s, xq, sx, stream=None):
    M, K = x.shape
    _check("sq_quant_act",
           lib().sq_quant_act(_ptr(x), _dtype_code(x), M, K, _ptr(s), _ptr(xq), _ptr(sx),
                              _stream(stream)))


def sq_fold_gamma(gamma, s, g, stream=None):
    K = gamma.shape[0]
    _check("sq_fold_gamma", lib().sq_fold_gamma(_ptr(gamma), _ptr(s), K, _ptr(g), _stream(stream)))


def sq_rmsnorm_quant(h, g, eps, xq, sx, rinv=None, stream=None):
    M, K = h.shape
    _check("sq_rmsnorm_quant",
           lib().sq_rmsnorm_quant(_ptr(h), _dtype_code(h), M, K, _ptr(g), float(eps), _ptr(xq), _ptr(sx),
                                  None if rinv is None else _ptr(rinv), _stream(stream)))


def sq_silu_mul_quant(gu, s, xq, sx, h=None, stream=None):
    """gu [M, 2I] = [gate | up] rows; xq [M, I] int8 and sx [M] fp32 out; h [M, I]
    (gu's dtype) receives SiLU(gate) * up when given."""
    M, I2 = gu.shape
    _check("sq_silu_mul_quant",
           lib().sq_silu_mul_quant(_ptr(gu), _dtype_code(gu), M, I2 // 2, _ptr(s), _ptr(xq), _ptr(sx),
                                   None if h is None else _ptr(h), _stream(stream)))


def sq_gptq_hessian(x, s, H, stream=None):
    """H [K, K] fp64 = xh^T xh over the calibration tokens x [T, K] (xh = x / s)."""
    T, K = x.shape
    _check("sq_gptq_hessian", lib().sq_gptq_hessian(_ptr(x), _dtype_code(x), T, K, _ptr(s), _ptr(H), _stream(stream)))


def sq_gptq_factor(H, U, damp_frac=0.01, workspace=None, stream=None):
    """Damps H in place and writes U, the upper Cholesky factor of H^-1."""
    import torch

    K = H.shape[0]
    need = int(lib().sq_gptq_workspace_size(K))
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=H.device)
    _check("sq_gptq_factor", lib().sq_gptq_factor(_ptr(H), K, float(damp_frac), _ptr(U), _ptr(workspace),
                                                  workspace.numel() * workspace.element_size(), _stream(stream)))


def sq_gptq_quant_weight(w, s, U, wq, sw, stream=None):
    """GPTQ codes wq [N, K] and per-channel scales sw [N] of the smoothed weight."""
    N, K = w.shape
    _check("sq_gptq_quant_weight", lib().sq_gptq_quant_weight(_ptr(w), _dtype_code(w), N, K, _ptr(s), _ptr(U),
                                                              _ptr(wq), _ptr(sw), _stream(stream)))


def gptq_weight(xcal, w, s, damp_frac=0.01, stream=None):
    """GPTQ in place of prepare_weight's plain rounding: (wq, sw) for the
    smoothed weight w * s, with the Hessian from the calibration tokens xcal."""
    import torch

    K = w.shape[1]
    H = torch.empty(K, K, dtype=torch.float64, device=w.device)
    U = torch.empty_like(H)
    sq_gptq_hessian(xcal, s, H, stream)
    sq_gptq_factor(H, U, damp_frac, stream=stream)
    wq = torch.empty(w.shape, dtype=torch.int8, device=w.device)
    sw = torch.empty(w.shape[0], dtype=torch.float32, device=w.device)
    sq_gptq_quant_weight(w, s, U, wq, sw, stream)
    return wq, sw


def sq_w8a8_gemm(xq, sx, wq, sw, y, stream=None):
    M, K = xq.shape
    N = wq.shape[0]
    _check("sq_w8a8_gemm",
           lib().sq_w8a8_gemm(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y),
                              _dtype_code(y), _stream(stream)))


def sq_w8a8_gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().sq_w8a8_gemm_workspace_size(M, N, K))


def sq_w8a8_gemm_ws(xq, sx, wq, sw, y, workspace=None, stream=None):
    """sq_w8a8_gemm with a workspace (allocated here when not given)."""
    import torch

    M, K = xq.shape
    N = wq.shape[0]
    if workspace is None:
        workspace = torch.empty(sq_w8a8_gemm_workspace_size(M, N, K), dtype=torch.uint8, device=xq.device)
    _check("sq_w8a8_gemm_ws",
           lib().sq_w8a8_gemm_ws(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y), _dtype_code(y),
                                 _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)))


def sq_w8a8_gemm_s32(xq, wq, acc, stream=None):
    M, K = xq.shape
    N = wq.shape[0]
    _check("sq_w8a8_gemm_s32",
           lib().sq_w8a8_gemm_s32(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc), _stream(stream)))


def sq_linear_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().sq_linear_workspace_size(M, N, K))


def sq_linear(x, s, wq, sw, y, workspace=None, stream=None):
    M, K = x.shape
    N = wq.shape[0]
    ws_ptr = None if workspace is None else _ptr(workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("sq_linear",
           lib().sq_linear(_ptr(x), _dtype_code(x), _ptr(s), _ptr(wq), _ptr(sw), M, N, K, _ptr(y),
                           _dtype_code(y), ws_ptr, ws_bytes, _stream(stream)))


# bytes of the library's fixed scratch array used by sq_linear_noalloc
LINEAR_NOALLOC_SCRATCH_BYTES = 32 << 20


def sq_linear_noalloc(x, s, wq, sw, y, stream=None):
    """sq_linear with the library's own fixed scratch array instead of a
    caller workspace; allocates nothing.  Raises SQError(SQ_ERR_UNSUPPORTED)
    when sq_linear_workspace_size(M, N, K) exceeds
    LINEAR_NOALLOC_SCRATCH_BYTES."""
    M, K = x.shape
    N = wq.shape[0]
    _check("sq_linear_noalloc",
           lib().sq_linear_noalloc(_ptr(x), _dtype_code(x), _ptr(s), _ptr(wq), _ptr(sw), M, N, K,
                                   _ptr(y), _dtype_code(y), _stream(stream)))


def sq_device_status(stream=None) -> Tuple[int, int]:
    code = ctypes.c_uint32(0)
    st = lib().sq_device_status(_stream(stream), ctypes.byref(code))
    return st, int(code.value)


def sq_selftest_wait_timeout(limit_us: int, stream=None):
    _check("sq_selftest_wait_timeout", lib().sq_selftest_wait_timeout(int(limit_us), _stream(stream)))


# ---------------------------------------------------------------------------
# conveniences (allocate outputs with torch, then call the raw entry points)
# ---------------------------------------------------------------------------

def calibrate(x_batches, K: Optional[int] = None, stream=None):
    """Accumulate the per-channel absmax A_j over one or more calibration batches."""
    torch = _torch()
    batches = [x_batches] if hasattr(x_batches, "shape") else list(x_batches)
    K = K or batches[0].shape[1]
    ax = torch.zeros(K, dtype=torch.float32, device=batches[0].device)
    for b in batches:
        sq_calib_absmax(b, ax, stream)
    return ax


def prepare_weight(ax, w, alpha: float, stream=None):
    """Smoothing factors and the smoothed int8 weight: returns (s, wq, sw)."""
    torch = _torch()
    N, K = w.shape
    s = torch.empty(K, dtype=torch.float32, device=w.device)
    sq_smooth_factors(ax, w, alpha, s, None, stream)
    wq = torch.empty(N, K, dtype=torch.int8, device=w.device)
    sw = torch.empty(N, dtype=torch.float32, device=w.device)
    sq_smooth_quant_weight(w, s, wq, sw, stream)
    return s, wq, sw


def linear(x, s, wq, sw, out_dtype=None, workspace=None, stream=None):
    """Y = dequant(quant(X / s) @ Wq^T) with a torch-allocated output."""
    torch = _torch()
    M, K = x.shape
    N = wq.shape[0]
    y = torch.empty(M, N, dtype=out_dtype or x.dtype, device=x.device)
    need = sq_linear_workspace_size(M, N, K)
    if need and (workspace is None or workspace.numel() * workspace.element_size() < need):
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    sq_linear(x, s, wq, sw, y, workspace if need else None, stream)
    return y

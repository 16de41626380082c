"""NumPy front end of the plain C oracle (``sq_oracle.c``).

TEST INFRASTRUCTURE ONLY: the test-suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product path (the CUDA
library and its Python binding) never imports this module.

Every function takes and returns NumPy arrays.  bf16 tensors travel as their
raw 16-bit patterns (``np.uint16``); fp32 as ``np.float32``.  The arithmetic is
all in the C file; this module only marshals arguments, except for
``smoothing_identity_fp64`` and ``fp64_reference_linear``, which are plain fp64
restatements used for the quantisation-error report and the identity check.

Sources (page title and section):
  * "Understanding W8A8 INT8 LLM Quantization": "Why Naive Weight Quantization
    Doesn't Work, and How GPTQ Fixes It" (per-channel weight scale and
    rounding), "Why Activation Quantization Is Hard, and How SmoothQuant Fixes
    It" (per-token dynamic scale), "Where the outlier actually comes from" and
    "How the smoothing factor is computed" (smoothing);
  * "quant_llm_int8": "The architecture: every piece explained" (int32
    accumulation, outer-product dequantisation).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_LIB = os.path.join(_HERE, "libsqoracle.so")
_lock = threading.Lock()
_lib = None

F32 = 0
BF16 = 1

GCC_FLAGS = ["-O2", "-fPIC", "-shared", "-ffp-contract=off", "-fopenmp", "-Wall"]


def build(force: bool = False) -> str:
    """Compile ``sq_oracle.c`` into ``libsqoracle.so`` (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            P = ctypes.c_void_p
            I = ctypes.c_int64
            lib.sqo_calib_absmax.argtypes = [P, ctypes.c_int, I, I, I, P]
            lib.sqo_weight_in_absmax.argtypes = [P, ctypes.c_int, I, I, P]
            lib.sqo_smooth_factors.argtypes = [P, P, I, ctypes.c_float, P]
            lib.sqo_smooth_quant_weight.argtypes = [P, ctypes.c_int, I, I, P, P, P]
            lib.sqo_quant_act_rows.argtypes = [P, ctypes.c_int, I, I, P, P, I, P, P]
            lib.sqo_quant_act.argtypes = [P, ctypes.c_int, I, I, P, P, P]
            lib.sqo_gemm_i32.argtypes = [P, P, I, I, I, P]
            lib.sqo_gemm_i32_pairs.argtypes = [P, I, P, I, P, P, I, P]
            lib.sqo_dequant.argtypes = [P, P, P, I, I, P, P]
            lib.sqo_dequant_pairs.argtypes = [P, P, P, I, P, P]
            lib.sqo_fold_gamma.argtypes = [P, P, I, P]
            lib.sqo_rmsnorm_quant.argtypes = [P, ctypes.c_int, I, I, P, ctypes.c_float, ctypes.c_double, P, P, P,
                                              P, P, P, P]
            lib.sqo_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.sqo_gptq_hessian.argtypes = [P, ctypes.c_int, I, I, P, P]
            lib.sqo_gptq_damp.argtypes = [P, I, ctypes.c_float]
            lib.sqo_gptq_factor.argtypes = [P, I, P]
            lib.sqo_gptq_factor.restype = ctypes.c_int
            lib.sqo_gptq_quant_weight.argtypes = [P, ctypes.c_int, I, I, P, P, ctypes.c_double, P, P, P]
            lib.sqo_exp_f32.argtypes = [ctypes.c_float]
            lib.sqo_exp_f32.restype = ctypes.c_float
            lib.sqo_silu_f32.argtypes = [ctypes.c_float]
            lib.sqo_silu_f32.restype = ctypes.c_float
            lib.sqo_exp_silu_vec.argtypes = [P, I, ctypes.c_int, P]
            lib.sqo_silu_mul_quant.argtypes = [P, ctypes.c_int, I, I, P, P, P, P]
            lib.sqo_f32_to_bf16.restype = ctypes.c_uint16
            lib.sqo_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dt(a: np.ndarray) -> int:
    if a.dtype == np.float32:
        return F32
    if a.dtype == np.uint16:
        return BF16
    raise TypeError(f"oracle inputs are float32 or bf16 bit patterns (uint16), got {a.dtype}")


def _c(a, dtype=None):
    a = np.asarray(a) if dtype is None else np.asarray(a, dtype=dtype)
    return np.ascontiguousarray(a)


def num_threads() -> int:
    return int(_load().sqo_num_threads())


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32 (the bits become the high half)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round-half-to-even of fp32 values to bf16 bit patterns (the C routine, per element)."""
    lib = _load()
    flat = np.asarray(x, dtype=np.float32).ravel()
    out = np.fromiter((lib.sqo_f32_to_bf16(float(v)) for v in flat), dtype=np.uint16, count=flat.size)
    return out.reshape(np.shape(x))


def calib_absmax(x: np.ndarray) -> np.ndarray:
    """ax[j] = max_t |X[t, j]| for X [T, K] (fp32 or bf16 bits)."""
    x = _c(x)
    T, K = x.shape
    ax = np.empty(K, np.float32)
    _load().sqo_calib_absmax(_ptr(x), _dt(x), T, K, K, _ptr(ax))
    return ax


def weight_in_absmax(w: np.ndarray) -> np.ndarray:
    """aw[j] = max_n |W[n, j]| for W [N, K] (out x in)."""
    w = _c(w)
    N, K = w.shape
    aw = np.empty(K, np.float32)
    _load().sqo_weight_in_absmax(_ptr(w), _dt(w), N, K, _ptr(aw))
    return aw


def smooth_factors(ax: np.ndarray, aw: np.ndarray, alpha: float) -> np.ndarray:
    ax = _c(ax, np.float32)
    aw = _c(aw, np.float32)
    assert ax.shape == aw.shape and ax.ndim == 1
    s = np.empty_like(ax)
    _load().sqo_smooth_factors(_ptr(ax), _ptr(aw), ax.size, float(np.float32(alpha)), _ptr(s))
    return s


def smooth_quant_weight(w: np.ndarray, s: np.ndarray):
    """Returns (wq int8 [N, K], sw fp32 [N])."""
    w = _c(w)
    s = _c(s, np.float32)
    N, K = w.shape
    assert s.shape == (K,)
    wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    _load().sqo_smooth_quant_weight(_ptr(w), _dt(w), N, K, _ptr(s), _ptr(wq), _ptr(sw))
    return wq, sw


def quant_act(x: np.ndarray, s: np.ndarray, rows=None):
    """Returns (xq int8 [R, K], sx fp32 [R]) for all rows, or for the listed rows."""
    x = _c(x)
    s = _c(s, np.float32)
    M, K = x.shape
    assert s.shape == (K,)
    if rows is None:
        r = None
        R = M
    else:
        r = _c(rows, np.int64)
        assert r.ndim == 1 and (r.size == 0 or (r.min() >= 0 and r.max() < M))
        R = r.size
    xq = np.empty((R, K), np.int8)
    sx = np.empty(R, np.float32)
    _load().sqo_quant_act_rows(_ptr(x), _dt(x), K, K, _ptr(s), _ptr(r), R, _ptr(xq), _ptr(sx))
    return xq, sx


def fold_gamma(gamma: np.ndarray, s: np.ndarray) -> np.ndarray:
    """g = gamma / s per channel (fp32): RMSNorm's gamma with the smoothing folded in."""
    gamma = _c(gamma, np.float32)
    s = _c(s, np.float32)
    assert gamma.shape == s.shape and gamma.ndim == 1
    g = np.empty_like(gamma)
    _load().sqo_fold_gamma(_ptr(gamma), _ptr(s), gamma.size, _ptr(g))
    return g


def rmsnorm_quant(h: np.ndarray, g: np.ndarray, eps: float):
    """RMSNorm of each token row with the folded gamma g, then per-token int8
    quantisation.  Returns (xq int8 [M, K], sx fp32 [M], rinv fp32 [M])."""
    c = rmsnorm_quant_candidates(h, g, eps)
    return c["xq"], c["sx"], c["rinv"]


def rmsnorm_quant_candidates(h: np.ndarray, g: np.ndarray, eps: float, window: float = -1.0):
    """The RMSNorm quantiser's result, plus, for every token whose fp64 1/RMS
    lies within ``window`` (relative; negative: the summation-order bound
    (K + 16) 2^-52) of an fp32 rounding midpoint, the whole result for the
    fp32 neighbour across that midpoint.  Returns a dict of numpy arrays:
    xq, sx, rinv (the result), near (bool [M], flagged tokens), and xq_alt,
    sx_alt, rinv_alt (the alternate result; equal to the result where not
    flagged)."""
    h = _c(h)
    g = _c(g, np.float32)
    M, K = h.shape
    assert g.shape == (K,)
    out = {"xq": np.empty((M, K), np.int8), "sx": np.empty(M, np.float32), "rinv": np.empty(M, np.float32),
           "near": np.empty(M, np.uint8), "xq_alt": np.empty((M, K), np.int8), "sx_alt": np.empty(M, np.float32),
           "rinv_alt": np.empty(M, np.float32)}
    _load().sqo_rmsnorm_quant(_ptr(h), _dt(h), M, K, _ptr(g), float(eps), float(window), _ptr(out["xq"]),
                              _ptr(out["sx"]), _ptr(out["rinv"]), _ptr(out["near"]), _ptr(out["xq_alt"]),
                              _ptr(out["sx_alt"]), _ptr(out["rinv_alt"]))
    out["near"] = out["near"].astype(bool)
    return out


def exp_f32(x: np.ndarray) -> np.ndarray:
    """e^x per element by the fixed fp32 sequence of ``sqo_exp_f32``."""
    x = _c(x, np.float32)
    y = np.empty_like(x)
    _load().sqo_exp_silu_vec(_ptr(x), x.size, 0, _ptr(y))
    return y


def silu_f32(x: np.ndarray) -> np.ndarray:
    """SiLU(x) = x / (1 + e^-x) per element in fp32 (``sqo_silu_f32``)."""
    x = _c(x, np.float32)
    y = np.empty_like(x)
    _load().sqo_exp_silu_vec(_ptr(x), x.size, 1, _ptr(y))
    return y


def silu_mul_quant(gu: np.ndarray, s: np.ndarray):
    """Gated feed-forward activation h = SiLU(gate) * up (gu = [gate | up], [M, 2I]),
    rounded to gu's storage type, then per-token int8 quantisation of h / s.
    Returns (xq int8 [M, I], sx fp32 [M], h fp32 [M, I])."""
    gu = _c(gu)
    s = _c(s, np.float32)
    M, I2 = gu.shape
    assert I2 % 2 == 0
    I = I2 // 2
    assert s.shape == (I,)
    xq = np.empty((M, I), np.int8)
    sx = np.empty(M, np.float32)
    h = np.empty((M, I), np.float32)
    _load().sqo_silu_mul_quant(_ptr(gu), _dt(gu), M, I, _ptr(s), _ptr(xq), _ptr(sx), _ptr(h))
    return xq, sx, h


def gptq_hessian(x: np.ndarray, s: np.ndarray) -> np.ndarray:
    """H = sum_t xh_t xh_t^T in fp64 (xh = X / s per element in fp32), [K, K]."""
    x = _c(x)
    s = _c(s, np.float32)
    T, K = x.shape
    H = np.empty((K, K), np.float64)
    _load().sqo_gptq_hessian(_ptr(x), _dt(x), T, K, _ptr(s), _ptr(H))
    return H


def gptq_damp(H: np.ndarray, damp_frac: float) -> np.ndarray:
    """A damped copy of H: damp_frac times the mean diagonal added to the diagonal."""
    Hd = np.array(H, np.float64, order="C", copy=True)
    _load().sqo_gptq_damp(_ptr(Hd), Hd.shape[0], float(damp_frac))
    return Hd


def gptq_factor(H: np.ndarray) -> np.ndarray:
    """U, the upper Cholesky factor of H^-1 (H^-1 = U^T U); raises if H is not
    positive definite."""
    H = _c(H, np.float64)
    K = H.shape[0]
    U = np.empty((K, K), np.float64)
    if _load().sqo_gptq_factor(_ptr(H), K, _ptr(U)) != 0:
        raise ValueError("H is not positive definite")
    return U


def gptq_quant_weight(w: np.ndarray, s: np.ndarray, U: np.ndarray):
    """GPTQ codes and per-channel scales of the smoothed weight W * s:
    (wq int8 [N, K], sw fp32 [N])."""
    wq, sw, _ = gptq_quant_weight_ties(w, s, U)
    return wq, sw


def gptq_quant_weight_ties(w: np.ndarray, s: np.ndarray, U: np.ndarray, tau: float = 2.0 ** -20):
    """As gptq_quant_weight, plus per row the first weight index whose
    quotient lies within tau of a rounding tie (-1 if none): (wq, sw, tie_pos)."""
    w = _c(w)
    s = _c(s, np.float32)
    U = _c(U, np.float64)
    N, K = w.shape
    wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    tie = np.empty(N, np.int64)
    _load().sqo_gptq_quant_weight(_ptr(w), _dt(w), N, K, _ptr(s), _ptr(U), float(tau), _ptr(wq), _ptr(sw),
                                  _ptr(tie))
    return wq, sw, tie


def gptq(xcal: np.ndarray, w: np.ndarray, s: np.ndarray, damp_frac: float = 0.01):
    """The whole GPTQ weight rounding: Hessian, damping, factor, rows."""
    U = gptq_factor(gptq_damp(gptq_hessian(xcal, s), damp_frac))
    wq, sw = gptq_quant_weight(w, s, U)
    return wq, sw, U


def gemm_i32(xq: np.ndarray, wq: np.ndarray) -> np.ndarray:
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    M, K = xq.shape
    N, K2 = wq.shape
    assert K == K2
    acc = np.empty((M, N), np.int32)
    _load().sqo_gemm_i32(_ptr(xq), _ptr(wq), M, N, K, _ptr(acc))
    return acc


def gemm_i32_pairs(xq: np.ndarray, wq: np.ndarray, ms, ns) -> np.ndarray:
    """acc for each (ms[i], ns[i]); xq rows are indexed by ms, wq rows by ns."""
    xq = _c(xq, np.int8)
    wq = _c(wq, np.int8)
    ms = _c(ms, np.int64)
    ns = _c(ns, np.int64)
    K = xq.shape[1]
    assert wq.shape[1] == K and ms.shape == ns.shape
    acc = np.empty(ms.size, np.int32)
    _load().sqo_gemm_i32_pairs(_ptr(xq), K, _ptr(wq), K, _ptr(ms), _ptr(ns), ms.size, _ptr(acc))
    return acc


def dequant(acc: np.ndarray, sx: np.ndarray, sw: np.ndarray, out: str = "f32") -> np.ndarray:
    """y = ((float)acc * sx[m]) * sw[n]; out = 'f32' or 'bf16' (bit patterns)."""
    acc = _c(acc, np.int32)
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    M, N = acc.shape
    yf = np.empty((M, N), np.float32) if out == "f32" else None
    yb = np.empty((M, N), np.uint16) if out == "bf16" else None
    _load().sqo_dequant(_ptr(acc), _ptr(sx), _ptr(sw), M, N, _ptr(yf), _ptr(yb))
    return yf if out == "f32" else yb


def dequant_pairs(acc, sx, sw, out: str = "f32") -> np.ndarray:
    acc = _c(acc, np.int32)
    sx = _c(sx, np.float32)
    sw = _c(sw, np.float32)
    n = acc.size
    assert sx.size == n and sw.size == n
    yf = np.empty(n, np.float32) if out == "f32" else None
    yb = np.empty(n, np.uint16) if out == "bf16" else None
    _load().sqo_dequant_pairs(_ptr(acc), _ptr(sx), _ptr(sw), n, _ptr(yf), _ptr(yb))
    return yf if out == "f32" else yb


def linear(x: np.ndarray, s: np.ndarray, wq: np.ndarray, sw: np.ndarray, out: str = "f32"):
    """The online path end to end: per-token quant of X/s, int32 GEMM, dequant."""
    xq, sx = quant_act(x, s)
    acc = gemm_i32(xq, wq)
    return dequant(acc, sx, sw, out), xq, sx, acc


def prepare(xcal: np.ndarray, w: np.ndarray, alpha: float):
    """The offline path: calibration absmax, smoothing factors, smoothed int8 weights."""
    ax = calib_absmax(xcal)
    aw = weight_in_absmax(w)
    s = smooth_factors(ax, aw, alpha)
    wq, sw = smooth_quant_weight(w, s)
    return ax, aw, s, wq, sw


# ---------------------------------------------------------------------------
# fp64 restatements (reporting and identity checks only)
# ---------------------------------------------------------------------------

def _as_f64(a: np.ndarray) -> np.ndarray:
    a = np.asarray(a)
    if a.dtype == np.uint16:
        a = bf16_bits_to_f32(a)
    return a.astype(np.float64)


def smoothing_identity_fp64(x, w, s):
    """(X diag(s)^-1)(W diag(s))^T and X W^T, both in fp64.

    "Where the outlier actually comes from": dividing the activation channel by
    s and multiplying the matching weight input channel by s leaves the layer's
    output unchanged.
    """
    X = _as_f64(x)
    W = _as_f64(w)
    S = np.asarray(s, dtype=np.float64)
    return (X / S[None, :]) @ (W * S[None, :]).T, X @ W.T


def fp64_reference_linear(x, w) -> np.ndarray:
    """Unquantised X W^T in fp64 (for the reported quantisation error only)."""
    return _as_f64(x) @ _as_f64(w).T

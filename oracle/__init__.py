"""CPU oracle for the SmoothQuant W8A8 linear layer -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference leg
of ``bench.py`` may import this package.  The product path (the CUDA library)
neither imports it nor shares code with it.

The arithmetic lives in ``sq_oracle.c`` (plain loops, IEEE binary32 with one
rounding per written operation); this module only marshals numpy arrays into it
and adds the binary64 definitions the pins need (the exact smoothing identity and
the unquantised linear).  bfloat16 arrays are passed around as ``numpy.uint16``
bit patterns.

Sources (page title, section):
  * "4.2 W8A8 量化与 SmoothQuant" sec. 3-4 (equivalence Y = (X diag(s)^-1)(diag(s) W),
    s_j = max|X_j|^a / max|W_j|^(1-a)), sec. 6 (LayerNorm folding), sec. 7.1 (per-channel
    static weights, per-token dynamic activations).
  * "量化：只压权重，与训练后量化（PTQ）", SmoothQuant section (W_j = row j of W;
    worked 3x3 example).
  * "SmoothQuant大模型平滑量化技术", Python demo (symmetric INT8: max/127, round, clip).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

F32, BF16, I32 = 0, 1, 2

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P, I64, I, F = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        L.sqo_calib_absmax.argtypes = [P, I, I64, I64, I64, I, I, P]
        L.sqo_calib_absmax.restype = None
        L.sqo_smooth_factors.argtypes = [P, P, I64, F, P]
        L.sqo_smooth_factors.restype = None
        L.sqo_fold_quant_weights.argtypes = [P, I, I64, I64, I64, P, P, P, P, P, P, P]
        L.sqo_fold_quant_weights.restype = None
        L.sqo_layernorm.argtypes = [P, I, I64, I64, I64, P, P, F, P]
        L.sqo_layernorm.restype = None
        L.sqo_calib_ln_absmax.argtypes = [P, I, I64, I64, I64, P, P, F, I, P]
        L.sqo_calib_ln_absmax.restype = None
        L.sqo_ln_smooth_quant.argtypes = [P, I, I64, I64, I64, P, P, P, F, P, P]
        L.sqo_ln_smooth_quant.restype = None
        L.sqo_ln_smooth_quant_per_tensor.argtypes = [P, I, I64, I64, I64, P, P, P, F, I, P, P, P]
        L.sqo_ln_smooth_quant_per_tensor.restype = None
        L.sqo_quant_per_tensor.argtypes = [P, I64, P, P]
        L.sqo_quant_per_tensor.restype = None
        L.sqo_w8a8_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, I, I64]
        L.sqo_w8a8_gemm.restype = I64
        L.sqo_fold_next_smoothing.argtypes = [P, P, I64, P]
        L.sqo_fold_next_smoothing.restype = None
        L.sqo_e4m3_encode.argtypes = [F]
        L.sqo_e4m3_encode.restype = ctypes.c_uint8
        L.sqo_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.sqo_e4m3_decode.restype = F
        L.sqo_fold_quant_weights_fp8.argtypes = [P, I, I64, I64, I64, P, P, P, P, P, P, P]
        L.sqo_fold_quant_weights_fp8.restype = None
        L.sqo_ln_smooth_quant_fp8.argtypes = [P, I, I64, I64, I64, P, P, P, F, P, P]
        L.sqo_ln_smooth_quant_fp8.restype = None
        L.sqo_fp8_gemm.argtypes = [P, P, P, P, I64, I64, I64, P, P, I, I64]
        L.sqo_fp8_gemm.restype = None
        L.sqo_f32_to_bf16.argtypes = [F]
        L.sqo_f32_to_bf16.restype = ctypes.c_uint16
        L.sqo_num_threads.argtypes = []
        L.sqo_num_threads.restype = I
        L.sqo_set_num_threads.argtypes = [I]
        L.sqo_set_num_threads.restype = None
        _lib = L
    return _lib


def num_threads() -> int:
    """Threads the oracle's OpenMP loops use (OMP_NUM_THREADS or all cores)."""
    return lib().sqo_num_threads()


def set_num_threads(n: int) -> None:
    """Threads for the oracle's following parallel loops (results do not depend on it)."""
    lib().sqo_set_num_threads(int(n))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _dtype_code(x: np.ndarray) -> int:
    if x.dtype == np.uint16:
        return BF16
    if x.dtype == np.float32:
        return F32
    raise TypeError(f"oracle inputs are float32 or bfloat16 bits (uint16), got {x.dtype}")


def _c(x, dtype=None):
    if x is None:
        return None
    return np.ascontiguousarray(x if dtype is None else x.astype(dtype, copy=False))


# ----------------------------------------------------------------------------- bf16 helpers
def bf16_to_f32(u16: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.asarray(u16, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 bits, nearest-even (element-wise through the C routine)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    f = lib().sqo_f32_to_bf16
    out = np.empty(x.shape, dtype=np.uint16)
    flat_in, flat_out = x.reshape(-1), out.reshape(-1)
    for i in range(flat_in.size):
        flat_out[i] = f(float(flat_in[i]))
    return out


# ----------------------------------------------------------------------------- method steps
def calib_absmax(x: np.ndarray, axis: int, out: np.ndarray | None = None) -> np.ndarray:
    """axis 0: per-column max |x| (per input channel over tokens); axis 1: per-row max |x|.

    ``out`` given: running max folded into it (accumulate mode)."""
    x = _c(x)
    rows, cols = x.shape
    n = cols if axis == 0 else rows
    acc = out is not None
    res = np.zeros(n, np.float32) if out is None else np.array(out, dtype=np.float32, copy=True)
    lib().sqo_calib_absmax(_ptr(x), _dtype_code(x), rows, cols, cols, axis, int(acc), _ptr(res))
    return res


def smooth_factors(ax: np.ndarray, aw: np.ndarray, alpha: float) -> np.ndarray:
    """s_j = ax_j^alpha / aw_j^(1-alpha), rounded once to float32."""
    ax, aw = _c(ax, np.float32), _c(aw, np.float32)
    s = np.empty(ax.shape[0], np.float32)
    lib().sqo_smooth_factors(_ptr(ax), _ptr(aw), ax.shape[0], float(alpha), _ptr(s))
    return s


def fold_quant_weights(W: np.ndarray, s: np.ndarray, gamma=None, beta=None):
    """W [K, N] (row j = input channel) -> (Wq [N, K] int8, sw [N], gamma', beta')."""
    W, s = _c(W), _c(s, np.float32)
    K, N = W.shape
    wq = np.empty((N, K), np.int8)
    sw = np.empty(N, np.float32)
    gamma, beta = _c(gamma, np.float32), _c(beta, np.float32)
    gf = np.empty(K, np.float32) if gamma is not None else None
    bf = np.empty(K, np.float32) if beta is not None else None
    lib().sqo_fold_quant_weights(_ptr(W), _dtype_code(W), K, N, N, _ptr(s), _ptr(gamma), _ptr(beta),
                                 _ptr(wq), _ptr(sw), _ptr(gf), _ptr(bf))
    return wq, sw, gf, bf


def layernorm(x: np.ndarray, gamma: np.ndarray, beta=None, eps: float = 1e-5) -> np.ndarray:
    """LayerNorm rows in float32 with the fixed statistic order of the C oracle."""
    x = _c(x)
    M, K = x.shape
    y = np.empty((M, K), np.float32)
    lib().sqo_layernorm(_ptr(x), _dtype_code(x), M, K, K, _ptr(_c(gamma, np.float32)),
                        _ptr(_c(beta, np.float32)), float(eps), _ptr(y))
    return y


def calib_ln_absmax(x: np.ndarray, gamma, beta=None, eps: float = 1e-5, out=None) -> np.ndarray:
    """max_i |LN(x_i)_j| with the original gamma, beta (beta may be None)."""
    x = _c(x)
    M, K = x.shape
    acc = out is not None
    res = np.zeros(K, np.float32) if out is None else np.array(out, dtype=np.float32, copy=True)
    lib().sqo_calib_ln_absmax(_ptr(x), _dtype_code(x), M, K, K, _ptr(_c(gamma, np.float32)),
                              _ptr(_c(beta, np.float32)), float(eps), int(acc), _ptr(res))
    return res


def ln_smooth_quant(x: np.ndarray, gamma_f=None, beta_f=None, s=None, eps: float = 1e-5):
    """Per-token INT8 of LN(x) with folded gamma'/beta' (LN mode) or of x / s (plain mode)."""
    if (gamma_f is None) == (s is None):
        raise ValueError("exactly one of gamma_f (LayerNorm mode) and s (plain mode) is given")
    x = _c(x)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    lib().sqo_ln_smooth_quant(_ptr(x), _dtype_code(x), M, K, K, _ptr(_c(gamma_f, np.float32)),
                              _ptr(_c(beta_f, np.float32)), _ptr(_c(s, np.float32)), float(eps),
                              _ptr(xq), _ptr(sx))
    return xq, sx


def ln_smooth_quant_per_tensor(x: np.ndarray, gamma_f=None, beta_f=None, s=None, eps: float = 1e-5,
                               static_scale: float | None = None):
    """One scale for the whole tensor: max|y|/127 (dynamic) or the given calibrated scale
    (static, values beyond it clamp to +-127).  Returns (xq, sx [every row = scale], scale)."""
    if (gamma_f is None) == (s is None):
        raise ValueError("exactly one of gamma_f (LayerNorm mode) and s (plain mode) is given")
    x = _c(x)
    M, K = x.shape
    xq = np.empty((M, K), np.int8)
    sx = np.empty(M, np.float32)
    sc = np.array([0.0 if static_scale is None else static_scale], np.float32)
    lib().sqo_ln_smooth_quant_per_tensor(_ptr(x), _dtype_code(x), M, K, K, _ptr(_c(gamma_f, np.float32)),
                                         _ptr(_c(beta_f, np.float32)), _ptr(_c(s, np.float32)), float(eps),
                                         int(static_scale is not None), _ptr(sc), _ptr(xq), _ptr(sx))
    return xq, sx, float(sc[0])


def quant_per_tensor(y: np.ndarray):
    """One scale max|y|/127 for the whole tensor; returns (codes, scale)."""
    y = _c(y, np.float32)
    q = np.empty(y.shape, np.int8)
    sc = np.zeros(1, np.float32)
    lib().sqo_quant_per_tensor(_ptr(y), y.size, _ptr(q), _ptr(sc))
    return q, float(sc[0])


def w8a8_gemm(xq: np.ndarray, sx: np.ndarray, wq: np.ndarray, sw: np.ndarray, out: str = "bf16"):
    """acc = xq @ wq^T exactly; out 'i32' -> acc, 'f32' -> (acc*sx)*sw, 'bf16' -> its bf16 bits."""
    xq, wq = _c(xq, np.int8), _c(wq, np.int8)
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError("xq and wq disagree on K")
    code, dt = {"i32": (I32, np.int32), "f32": (F32, np.float32), "bf16": (BF16, np.uint16)}[out]
    y = np.empty((M, N), dt)
    sx_, sw_ = _c(sx, np.float32), _c(sw, np.float32)
    over = lib().sqo_w8a8_gemm(_ptr(xq), _ptr(sx_), _ptr(wq), _ptr(sw_), M, N, K, _ptr(y), code, N)
    if over:
        raise OverflowError(f"{over} accumulators outside int32")
    return y


def fold_next_smoothing(sw: np.ndarray, s_next: np.ndarray) -> np.ndarray:
    """sw / s_next in binary32: the next linear's smoothing folded into this linear's scales."""
    sw, s_next = _c(sw, np.float32), _c(s_next, np.float32)
    out = np.empty_like(sw)
    lib().sqo_fold_next_smoothing(_ptr(sw), _ptr(s_next), sw.size, _ptr(out))
    return out


# ----------------------------------------------------------------------------- FP8 (E4M3) variant
def e4m3_encode(v) -> np.ndarray:
    """float32 values -> E4M3 codes (uint8): nearest even, saturating at +-448."""
    v = np.asarray(v, dtype=np.float32)
    f = lib().sqo_e4m3_encode
    return np.array([f(float(a)) for a in v.reshape(-1)], np.uint8).reshape(v.shape)


def e4m3_decode(c) -> np.ndarray:
    """E4M3 codes (uint8) -> float32 values (exact)."""
    c = np.asarray(c, dtype=np.uint8)
    f = lib().sqo_e4m3_decode
    return np.array([f(int(a)) for a in c.reshape(-1)], np.float32).reshape(c.shape)


def fold_quant_weights_fp8(W: np.ndarray, s: np.ndarray, gamma=None, beta=None):
    """W [K, N] -> (Wq [N, K] E4M3 codes, sw [N] = column max / 448, gamma', beta')."""
    W, s = _c(W), _c(s, np.float32)
    K, N = W.shape
    wq = np.empty((N, K), np.uint8)
    sw = np.empty(N, np.float32)
    gamma, beta = _c(gamma, np.float32), _c(beta, np.float32)
    gf = np.empty(K, np.float32) if gamma is not None else None
    bf = np.empty(K, np.float32) if beta is not None else None
    lib().sqo_fold_quant_weights_fp8(_ptr(W), _dtype_code(W), K, N, N, _ptr(s), _ptr(gamma), _ptr(beta),
                                     _ptr(wq), _ptr(sw), _ptr(gf), _ptr(bf))
    return wq, sw, gf, bf


def ln_smooth_quant_fp8(x: np.ndarray, gamma_f=None, beta_f=None, s=None, eps: float = 1e-5):
    """Per-token E4M3 of LN(x) (folded gamma', beta') or of x / s; sx = row max / 448."""
    if (gamma_f is None) == (s is None):
        raise ValueError("exactly one of gamma_f (LayerNorm mode) and s (plain mode) is given")
    x = _c(x)
    M, K = x.shape
    xq = np.empty((M, K), np.uint8)
    sx = np.empty(M, np.float32)
    lib().sqo_ln_smooth_quant_fp8(_ptr(x), _dtype_code(x), M, K, K, _ptr(_c(gamma_f, np.float32)),
                                  _ptr(_c(beta_f, np.float32)), _ptr(_c(s, np.float32)), float(eps),
                                  _ptr(xq), _ptr(sx))
    return xq, sx


def fp8_gemm(xq: np.ndarray, sx: np.ndarray, wq: np.ndarray, sw: np.ndarray, out: str = "bf16"):
    """Exact accumulators acc = dec(xq) @ dec(wq)^T (float64) and the output
    ((float)acc * sx) * sw as 'f32' or 'bf16' bits.  Returns (acc, y)."""
    xq, wq = _c(xq, np.uint8), _c(wq, np.uint8)
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError("xq and wq disagree on K")
    code, dt = {"f32": (F32, np.float32), "bf16": (BF16, np.uint16)}[out]
    acc = np.empty((M, N), np.float64)
    y = np.empty((M, N), dt)
    lib().sqo_fp8_gemm(_ptr(xq), _ptr(_c(sx, np.float32)), _ptr(wq), _ptr(_c(sw, np.float32)), M, N, K,
                       _ptr(acc), _ptr(y), code, N)
    return acc, y


# ----------------------------------------------------------------------------- alpha search
def alpha_grid(n: int = 20) -> np.ndarray:
    """n migration strengths evenly covering [0, 1] (both ends included)."""
    return np.linspace(0.0, 1.0, n).astype(np.float32)


def alpha_search(x: np.ndarray, W: np.ndarray, alphas, gamma=None, beta=None, eps: float = 1e-5):
    """Migration strength by grid search on calibration data.

    "4.2 W8A8 量化与 SmoothQuant" sec. 5.2: alpha is fixed once, offline, by a grid search on
    calibration samples; "量化：只压权重，与训练后量化（PTQ）", AWQ paragraph: the search
    objective is the layer-output error || Q(W diag(s)) (diag(s)^-1 X) - W X || over a grid
    of alpha in [0, 1].  (The paper's own criterion, validation perplexity, needs a model and
    data; the layer-output error is the objective the pages give for a data-only search.)

    For each alpha: s = smooth_factors(ax, aw, alpha) with ax the calibration absmax of the
    layer input (LN(x; gamma, beta) when gamma is given, else x) and aw the weight row absmax;
    the W8A8 layer of this oracle (fold, per-token quantiser, INT8 GEMM, binary32 epilogue
    ((float)acc * sx) * sw); err = ||Y_hat - Y||_F^2 / ||Y||_F^2 with Y = X_in W in float64.
    Returns err [len(alphas)] (float64)."""
    alphas = np.asarray(alphas, np.float32)
    x, W = _c(x), _c(W)
    if gamma is not None:
        x_in = layernorm(x, gamma, beta, eps)
        ax = calib_absmax(x_in, 0)
    else:
        x_in = bf16_to_f32(x) if x.dtype == np.uint16 else x
        ax = calib_absmax(x, 0)
    aw = calib_absmax(W, 1)
    W32 = bf16_to_f32(W) if W.dtype == np.uint16 else W
    Y = x_in.astype(np.float64) @ W32.astype(np.float64)
    den = float(np.sum(Y * Y))
    out = np.empty(alphas.size, np.float64)
    for i, a in enumerate(alphas):
        s = smooth_factors(ax, aw, float(a))
        wq, sw, gf, bf = fold_quant_weights(W, s, gamma, beta)
        xq, sx = ln_smooth_quant(x, gamma_f=gf, beta_f=bf, eps=eps) if gamma is not None else ln_smooth_quant(x, s=s)
        yh = w8a8_gemm(xq, sx, wq, sw, "f32").astype(np.float64)
        out[i] = float(np.sum((yh - Y) ** 2)) / den
    return out


# ----------------------------------------------------------------------------- binary64 definitions
def smooth_transform_f64(X: np.ndarray, W: np.ndarray, s: np.ndarray):
    """X' = X diag(s)^-1 (columns divided), W' = diag(s) W (rows scaled), in float64."""
    s64 = np.asarray(s, dtype=np.float64)
    return np.asarray(X, np.float64) / s64[None, :], s64[:, None] * np.asarray(W, np.float64)


def dequant_linear_f64(xq, sx, wq, sw) -> np.ndarray:
    """Y = (xq * sx[:, None]) @ (wq * sw[:, None])^T in float64 (the dequantised output)."""
    a = np.asarray(xq, np.float64) * np.asarray(sx, np.float64)[:, None]
    b = np.asarray(wq, np.float64) * np.asarray(sw, np.float64)[:, None]
    return a @ b.T

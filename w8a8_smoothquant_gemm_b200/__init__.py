"""SmoothQuant W8A8 linear layer for NVIDIA B200 (sm_100a) -- Python binding.

A thin ctypes layer over the C ABI in ``include/sq_w8a8.h`` (``libsq_w8a8.so``, built
in-tree by ``build.py``).  The functions keep the C names; they only marshal torch CUDA
tensors (device pointers, sizes, the current stream) and allocate outputs with torch's
allocator.  Every step runs in the library's CUDA kernels; there is no other code path:
if the library cannot be loaded, every call raises.

Pipeline ("4.2 W8A8 量化与 SmoothQuant", sec. 7.1):
  offline:  sq_calib_absmax / sq_calib_ln_absmax -> sq_smooth_factors -> sq_fold_quant_weights
  runtime:  sq_ln_smooth_quant -> sq_w8a8_gemm
FP8 (E4M3) variant of the quantised steps: sq_fold_quant_weights_fp8, sq_ln_smooth_quant_fp8,
sq_w8a8_gemm_fp8.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

SQ_F32, SQ_BF16, SQ_I32 = 0, 1, 2
SQ_MAX_K = 133136
SQ_MAX_K_ROW = 65536
_STATUS = {0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_UNSUPPORTED", 3: "SQ_ERR_ALIGNMENT",
           4: "SQ_ERR_CUDA", 5: "SQ_ERR_WORKSPACE"}

LIB_PATH = _build.LIB


class SQError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {_STATUS.get(status, status)}")
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded C library (built first if sources are newer).  Raises if unavailable."""
    global _lib
    if _lib is None:
        if not _build.up_to_date():
            _build.build()
        L = ctypes.CDLL(LIB_PATH)
        P, I64, I, F, SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        sigs = {
            "sq_calib_absmax": [P, I, I64, I64, I64, I, I, P, P],
            "sq_calib_ln_absmax": [P, I, I64, I64, I64, P, P, F, I, P, P],
            "sq_smooth_factors": [P, P, I64, F, P, P],
            "sq_fold_quant_weights": [P, I, I64, I64, I64, P, P, P, P, P, P, P, P],
            "sq_ln_smooth_quant": [P, I, I64, I64, I64, P, P, P, F, P, P, P],
            "sq_ln_smooth_quant_per_tensor": [P, I, I64, I64, I64, P, P, P, F, I, P, P, P, P],
            "sq_w8a8_gemm": [P, P, P, P, I64, I64, I64, P, I, I64, P, SZ, P],
            "sq_device_error": [P, I, P],
            "sq_fold_quant_weights_fp8": [P, I, I64, I64, I64, P, P, P, P, P, P, P, P],
            "sq_ln_smooth_quant_fp8": [P, I, I64, I64, I64, P, P, P, F, P, P, P],
            "sq_w8a8_gemm_fp8": [P, P, P, P, I64, I64, I64, P, I, I64, P, SZ, P],
            "sq_fold_next_smoothing": [P, P, I64, P, P],
            "sq_fold_kernel_launches": [P, I, I64, I64, I64],
            "sq_alpha_search": [P, I, I64, I64, I64, P, P, F, P, I, I64, I64, P, I, P, P, SZ, P],
            "sq_selfcheck_shared_divisor": [P, I64, P, I64, P, P, P],
            "sq_w8a8_gemm_rowmax": [P, P, P, P, I64, I64, I64, P, I, I64, P, P, SZ, P],
            "sq_quant_codes": [P, I, I64, I64, I64, P, P, P, P],
            "sq_set_wait_limit": [ctypes.c_uint64, P],
        }
        for name, argt in sigs.items():
            fn = getattr(L, name)
            fn.argtypes = argt
            fn.restype = ctypes.c_int
        L.sq_w8a8_gemm_workspace_size.argtypes = [I64, I64, I64]
        L.sq_w8a8_gemm_workspace_size.restype = SZ
        L.sq_alpha_search_workspace_size.argtypes = [I64, I64, I64]
        L.sq_alpha_search_workspace_size.restype = SZ
        L.sq_status_string.argtypes = [I]
        L.sq_status_string.restype = ctypes.c_char_p
        L.sq_abi_version.argtypes = []
        L.sq_abi_version.restype = I
        _lib = L
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise SQError(fn, status)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SQ_BF16
    if t.dtype == torch.float32:
        return SQ_F32
    raise TypeError(f"expected a bfloat16 or float32 tensor, got {t.dtype}")


def _mat(t: torch.Tensor, name: str) -> torch.Tensor:
    if t.dim() != 2 or not t.is_cuda:
        raise ValueError(f"{name} must be a 2-D CUDA tensor")
    if t.stride(1) != 1:
        raise ValueError(f"{name} must have unit column stride")
    return t


def _vec(t: torch.Tensor | None, n: int, name: str):
    if t is None:
        return None
    if t.dtype != torch.float32 or not t.is_cuda or t.numel() != n or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous float32 CUDA vector of {n} elements")
    return t


# ----------------------------------------------------------------------------- the five calls
def sq_calib_absmax(x: torch.Tensor, axis: int, out: torch.Tensor | None = None, accumulate: bool = False,
                    stream=None) -> torch.Tensor:
    """axis 0: out[j] = max_i |x[i, j]|; axis 1: out[i] = max_j |x[i, j]|."""
    x = _mat(x, "x")
    n = x.shape[1] if axis == 0 else x.shape[0]
    if out is None:
        out = torch.empty(n, dtype=torch.float32, device=x.device)
    _vec(out, n, "out")
    _check("sq_calib_absmax", lib().sq_calib_absmax(_ptr(x), _dt(x), x.shape[0], x.shape[1], x.stride(0), axis,
                                                    int(accumulate), _ptr(out), _stream(stream)))
    return out


def sq_calib_ln_absmax(x: torch.Tensor, gamma: torch.Tensor, beta: torch.Tensor | None = None, eps: float = 1e-5,
                       out: torch.Tensor | None = None, accumulate: bool = False, stream=None) -> torch.Tensor:
    """out[j] = max_i |LayerNorm(x_i)_j| with gamma, beta (beta may be None)."""
    x = _mat(x, "x")
    K = x.shape[1]
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=x.device)
    _vec(out, K, "out")
    _vec(gamma, K, "gamma")
    _vec(beta, K, "beta")
    _check("sq_calib_ln_absmax", lib().sq_calib_ln_absmax(_ptr(x), _dt(x), x.shape[0], K, x.stride(0), _ptr(gamma),
                                                          _ptr(beta), float(eps), int(accumulate), _ptr(out),
                                                          _stream(stream)))
    return out


def sq_smooth_factors(ax: torch.Tensor, aw: torch.Tensor, alpha: float, out: torch.Tensor | None = None,
                      stream=None) -> torch.Tensor:
    """s_j = ax_j^alpha / aw_j^(1 - alpha)."""
    K = ax.numel()
    _vec(ax, K, "ax")
    _vec(aw, K, "aw")
    if out is None:
        out = torch.empty(K, dtype=torch.float32, device=ax.device)
    _vec(out, K, "out")
    _check("sq_smooth_factors", lib().sq_smooth_factors(_ptr(ax), _ptr(aw), K, float(alpha), _ptr(out),
                                                        _stream(stream)))
    return out


def sq_fold_quant_weights(W: torch.Tensor, s: torch.Tensor, gamma: torch.Tensor | None = None,
                          beta: torch.Tensor | None = None, wq: torch.Tensor | None = None,
                          sw: torch.Tensor | None = None, gamma_f: torch.Tensor | None = None,
                          beta_f: torch.Tensor | None = None, stream=None):
    """W [K, N] -> (Wq [N, K] int8, sw [N], gamma / s or None, beta / s or None)."""
    W = _mat(W, "W")
    K, N = W.shape
    _vec(s, K, "s")
    _vec(gamma, K, "gamma")
    _vec(beta, K, "beta")
    dev = W.device
    if wq is None:
        wq = torch.empty(N, K, dtype=torch.int8, device=dev)
    if sw is None:
        sw = torch.empty(N, dtype=torch.float32, device=dev)
    gf = bf = None
    if gamma is not None:
        gf = gamma_f if gamma_f is not None else torch.empty(K, dtype=torch.float32, device=dev)
    if beta is not None:
        bf = beta_f if beta_f is not None else torch.empty(K, dtype=torch.float32, device=dev)
    _check("sq_fold_quant_weights",
           lib().sq_fold_quant_weights(_ptr(W), _dt(W), K, N, W.stride(0), _ptr(s), _ptr(gamma), _ptr(beta),
                                       _ptr(wq), _ptr(sw), _ptr(gf), _ptr(bf), _stream(stream)))
    return wq, sw, gf, bf


def sq_fold_next_smoothing(sw: torch.Tensor, s_next: torch.Tensor, out: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """sw / s_next: this linear's output scales with the next linear's smoothing folded in."""
    N = sw.shape[0]
    _vec(sw, N, "sw")
    _vec(s_next, N, "s_next")
    if out is None:
        out = torch.empty_like(sw)
    _check("sq_fold_next_smoothing", lib().sq_fold_next_smoothing(_ptr(sw), _ptr(s_next), N, _ptr(out),
                                                                  _stream(stream)))
    return out


def sq_ln_smooth_quant(x: torch.Tensor, gamma_f: torch.Tensor | None = None, beta_f: torch.Tensor | None = None,
                       s: torch.Tensor | None = None, eps: float = 1e-5, xq: torch.Tensor | None = None,
                       sx: torch.Tensor | None = None, stream=None):
    """LayerNorm mode (gamma_f given) or plain mode (s given) -> (xq [M, K] int8, sx [M])."""
    x = _mat(x, "x")
    M, K = x.shape
    _vec(gamma_f, K, "gamma_f")
    _vec(beta_f, K, "beta_f")
    _vec(s, K, "s")
    if xq is None:
        xq = torch.empty(M, K, dtype=torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    _check("sq_ln_smooth_quant", lib().sq_ln_smooth_quant(_ptr(x), _dt(x), M, K, x.stride(0), _ptr(gamma_f),
                                                          _ptr(beta_f), _ptr(s), float(eps), _ptr(xq), _ptr(sx),
                                                          _stream(stream)))
    return xq, sx


def sq_ln_smooth_quant_per_tensor(x: torch.Tensor, gamma_f: torch.Tensor | None = None,
                                  beta_f: torch.Tensor | None = None, s: torch.Tensor | None = None,
                                  eps: float = 1e-5, scale: torch.Tensor | None = None, static: bool = False,
                                  xq: torch.Tensor | None = None, sx: torch.Tensor | None = None, stream=None):
    """One scale for the whole tensor: dynamic (max|y|/127, written to `scale`) or static (the
    calibrated value in `scale`).  Returns (xq [M, K] int8, sx [M] = scale, scale [1])."""
    x = _mat(x, "x")
    M, K = x.shape
    _vec(gamma_f, K, "gamma_f")
    _vec(beta_f, K, "beta_f")
    _vec(s, K, "s")
    if scale is None:
        if static:
            raise ValueError("a static per-tensor scale must be given")
        scale = torch.empty(1, dtype=torch.float32, device=x.device)
    _vec(scale, 1, "scale")
    if xq is None:
        xq = torch.empty(M, K, dtype=torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    _check("sq_ln_smooth_quant_per_tensor",
           lib().sq_ln_smooth_quant_per_tensor(_ptr(x), _dt(x), M, K, x.stride(0), _ptr(gamma_f), _ptr(beta_f),
                                               _ptr(s), float(eps), int(static), _ptr(scale), _ptr(xq), _ptr(sx),
                                               _stream(stream)))
    return xq, sx, scale


def sq_fold_kernel_launches(W: torch.Tensor) -> int:
    """Kernels sq_fold_quant_weights(W, ...) launches (1, or 3 on the streaming route)."""
    W = _mat(W, "W")
    K, N = W.shape
    return int(lib().sq_fold_kernel_launches(_ptr(W), _dt(W), K, N, W.stride(0)))


def sq_w8a8_gemm_workspace_size(M: int, N: int, K: int) -> int:
    return int(lib().sq_w8a8_gemm_workspace_size(M, N, K))


_ODT = {torch.bfloat16: SQ_BF16, torch.float32: SQ_F32, torch.int32: SQ_I32}


def sq_w8a8_gemm(xq: torch.Tensor, sx: torch.Tensor | None, wq: torch.Tensor, sw: torch.Tensor | None,
                 out_dtype: torch.dtype = torch.bfloat16, y: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = bf16(((float)(xq @ wq^T) * sx[:, None]) * sw[None, :]) (or f32 / raw int32)."""
    if xq.dtype != torch.int8 or wq.dtype != torch.int8 or not xq.is_contiguous() or not wq.is_contiguous():
        raise ValueError("xq and wq must be contiguous int8 tensors")
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError("xq and wq disagree on K")
    if y is None:
        y = torch.empty(M, N, dtype=out_dtype, device=xq.device)
    ydt = _ODT[y.dtype]
    if ydt != SQ_I32:
        _vec(sx, M, "sx")
        _vec(sw, N, "sw")
    need = sq_w8a8_gemm_workspace_size(M, N, K)
    if workspace is None and need > 0:
        workspace = torch.zeros(need, dtype=torch.uint8, device=xq.device)  # its counters start at zero
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("sq_w8a8_gemm", lib().sq_w8a8_gemm(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y), ydt,
                                              y.stride(0), _ptr(workspace), ws_bytes, _stream(stream)))
    return y


def sq_w8a8_gemm_rowmax(xq: torch.Tensor, sx: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                        out_dtype: torch.dtype = torch.bfloat16, y: torch.Tensor | None = None,
                        rowmax: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    """sq_w8a8_gemm that also returns rowmax[m] = max_n |y[m, n]| of the stored outputs (the next
    linear's per-token statistic).  Returns (y, rowmax)."""
    if xq.dtype != torch.int8 or wq.dtype != torch.int8 or not xq.is_contiguous() or not wq.is_contiguous():
        raise ValueError("xq and wq must be contiguous int8 tensors")
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError("xq and wq disagree on K")
    if y is None:
        y = torch.empty(M, N, dtype=out_dtype, device=xq.device)
    if rowmax is None:
        rowmax = torch.empty(M, dtype=torch.float32, device=xq.device)
    _vec(sx, M, "sx")
    _vec(sw, N, "sw")
    _vec(rowmax, M, "rowmax")
    need = sq_w8a8_gemm_workspace_size(M, N, K)
    if workspace is None and need > 0:
        workspace = torch.zeros(need, dtype=torch.uint8, device=xq.device)  # its sums start at zero
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("sq_w8a8_gemm_rowmax", lib().sq_w8a8_gemm_rowmax(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y),
                                                            _ODT[y.dtype], y.stride(0), _ptr(rowmax), _ptr(workspace),
                                                            ws_bytes, _stream(stream)))
    return y, rowmax


def sq_quant_codes(x: torch.Tensor, rowmax: torch.Tensor, xq: torch.Tensor | None = None,
                   sx: torch.Tensor | None = None, stream=None):
    """Per-token INT8 codes of x given its row maxima: (xq [M, K] int8, sx [M] = rowmax / 127)."""
    x = _mat(x, "x")
    M, K = x.shape
    _vec(rowmax, M, "rowmax")
    if xq is None:
        xq = torch.empty(M, K, dtype=torch.int8, device=x.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    _check("sq_quant_codes", lib().sq_quant_codes(_ptr(x), _dt(x), M, K, x.stride(0), _ptr(rowmax), _ptr(xq), _ptr(sx),
                                                  _stream(stream)))
    return xq, sx


# ----------------------------------------------------------------------------- alpha search
def alpha_grid(n: int = 20) -> list:
    """n migration strengths evenly covering [0, 1] (both ends included)."""
    return [i / (n - 1) for i in range(n)] if n > 1 else [0.5]


def sq_alpha_search(x: torch.Tensor, W: torch.Tensor, alphas=None, gamma: torch.Tensor | None = None,
                    beta: torch.Tensor | None = None, eps: float = 1e-5, workspace: torch.Tensor | None = None,
                    stream=None):
    """Relative squared layer-output error of the W8A8 layer on the calibration batch x for each
    alpha (default: 20 values over [0, 1]).  Returns (err [n] float64 on the device, alphas)."""
    x = _mat(x, "x")
    W = _mat(W, "W")
    M, K = x.shape
    N = W.shape[1]
    if W.shape[0] != K:
        raise ValueError("x and W disagree on K")
    _vec(gamma, K, "gamma")
    _vec(beta, K, "beta")
    alphas = alpha_grid() if alphas is None else [float(a) for a in alphas]
    arr = (ctypes.c_float * len(alphas))(*alphas)
    err = torch.empty(len(alphas), dtype=torch.float64, device=x.device)
    need = int(lib().sq_alpha_search_workspace_size(M, K, N))
    if need == (1 << 64) - 1:
        raise ValueError("unsupported sizes for the alpha search")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check("sq_alpha_search",
           lib().sq_alpha_search(_ptr(x), _dt(x), M, K, x.stride(0), _ptr(gamma), _ptr(beta), float(eps), _ptr(W),
                                 _dt(W), N, W.stride(0), arr, len(alphas), _ptr(err), _ptr(workspace), ws_bytes,
                                 _stream(stream)))
    return err, alphas


# ----------------------------------------------------------------------------- FP8 (E4M3) variant
# Codes are uint8 tensors holding E4M3 bit patterns (view them as torch.float8_e4m3fn if
# wanted); scales are max / 448.
def sq_fold_quant_weights_fp8(W: torch.Tensor, s: torch.Tensor, gamma: torch.Tensor | None = None,
                              beta: torch.Tensor | None = None, wq: torch.Tensor | None = None,
                              sw: torch.Tensor | None = None, gamma_f: torch.Tensor | None = None,
                              beta_f: torch.Tensor | None = None, stream=None):
    """W [K, N] -> (Wq [N, K] E4M3 codes (uint8), sw [N], gamma / s or None, beta / s or None)."""
    W = _mat(W, "W")
    K, N = W.shape
    _vec(s, K, "s")
    _vec(gamma, K, "gamma")
    _vec(beta, K, "beta")
    dev = W.device
    if wq is None:
        wq = torch.empty(N, K, dtype=torch.uint8, device=dev)
    if sw is None:
        sw = torch.empty(N, dtype=torch.float32, device=dev)
    gf = bf = None
    if gamma is not None:
        gf = gamma_f if gamma_f is not None else torch.empty(K, dtype=torch.float32, device=dev)
    if beta is not None:
        bf = beta_f if beta_f is not None else torch.empty(K, dtype=torch.float32, device=dev)
    _check("sq_fold_quant_weights_fp8",
           lib().sq_fold_quant_weights_fp8(_ptr(W), _dt(W), K, N, W.stride(0), _ptr(s), _ptr(gamma), _ptr(beta),
                                           _ptr(wq), _ptr(sw), _ptr(gf), _ptr(bf), _stream(stream)))
    return wq, sw, gf, bf


def sq_ln_smooth_quant_fp8(x: torch.Tensor, gamma_f: torch.Tensor | None = None, beta_f: torch.Tensor | None = None,
                           s: torch.Tensor | None = None, eps: float = 1e-5, xq: torch.Tensor | None = None,
                           sx: torch.Tensor | None = None, stream=None):
    """LayerNorm mode (gamma_f given) or plain mode (s given) -> (xq [M, K] E4M3 codes, sx [M])."""
    x = _mat(x, "x")
    M, K = x.shape
    _vec(gamma_f, K, "gamma_f")
    _vec(beta_f, K, "beta_f")
    _vec(s, K, "s")
    if xq is None:
        xq = torch.empty(M, K, dtype=torch.uint8, device=x.device)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=x.device)
    _check("sq_ln_smooth_quant_fp8",
           lib().sq_ln_smooth_quant_fp8(_ptr(x), _dt(x), M, K, x.stride(0), _ptr(gamma_f), _ptr(beta_f), _ptr(s),
                                        float(eps), _ptr(xq), _ptr(sx), _stream(stream)))
    return xq, sx


def sq_w8a8_gemm_fp8(xq: torch.Tensor, sx: torch.Tensor, wq: torch.Tensor, sw: torch.Tensor,
                     out_dtype: torch.dtype = torch.bfloat16, y: torch.Tensor | None = None,
                     workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """y = bf16((acc * sx[:, None]) * sw[None, :]) with acc = dec(xq) @ dec(wq)^T in fp32 (or f32 y)."""
    if xq.dtype != torch.uint8 or wq.dtype != torch.uint8 or not xq.is_contiguous() or not wq.is_contiguous():
        raise ValueError("xq and wq must be contiguous uint8 tensors of E4M3 codes")
    M, K = xq.shape
    N = wq.shape[0]
    if wq.shape[1] != K:
        raise ValueError("xq and wq disagree on K")
    if y is None:
        y = torch.empty(M, N, dtype=out_dtype, device=xq.device)
    ydt = _ODT[y.dtype]
    _vec(sx, M, "sx")
    _vec(sw, N, "sw")
    need = sq_w8a8_gemm_workspace_size(M, N, K)
    if workspace is None and need > 0:
        workspace = torch.zeros(need, dtype=torch.uint8, device=xq.device)  # its counters start at zero
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check("sq_w8a8_gemm_fp8", lib().sq_w8a8_gemm_fp8(_ptr(xq), _ptr(sx), _ptr(wq), _ptr(sw), M, N, K, _ptr(y), ydt,
                                                      y.stride(0), _ptr(workspace), ws_bytes, _stream(stream)))
    return y


def sq_selfcheck_shared_divisor(a: torch.Tensor, b: torch.Tensor, want_quotients: bool = False, stream=None):
    """Checks the library's shared-divisor quotient against IEEE division for every pair
    (a[j], b[i]).  Returns ([scalar mismatches, packed mismatches, pairs checked] as a CUDA int64
    tensor, quotients [nb, na] or None)."""
    _vec(a, a.numel(), "a")
    _vec(b, b.numel(), "b")
    counts = torch.zeros(3, dtype=torch.int64, device=a.device)
    q = torch.empty(b.numel(), a.numel(), dtype=torch.float32, device=a.device) if want_quotients else None
    _check("sq_selfcheck_shared_divisor", lib().sq_selfcheck_shared_divisor(_ptr(a), a.numel(), _ptr(b), b.numel(),
                                                                            _ptr(q), _ptr(counts), _stream(stream)))
    return counts, q


WAIT_LIMIT_DEFAULT_NS = 10 * 1000 * 1000 * 1000


def sq_set_wait_limit(ns: int, stream=None) -> None:
    """Limit of the kernels' bounded waits on this device (0: every wait runs out at once)."""
    _check("sq_set_wait_limit", lib().sq_set_wait_limit(int(ns), _stream(stream)))


def sq_device_error(clear: bool = True, stream=None) -> int:
    """Device error word (non-zero when a kernel gave up on a bounded wait)."""
    code = ctypes.c_uint(0)
    _check("sq_device_error", lib().sq_device_error(ctypes.byref(code), int(clear), _stream(stream)))
    return code.value


def loaded_library_path() -> str:
    return os.path.realpath(LIB_PATH)

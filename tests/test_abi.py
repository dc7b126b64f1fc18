"""The C-ABI library builds for sm_100a, loads, exports every symbol its header declares,
and validates arguments on the host before touching the device.  CPU only: every call
below returns its status before any CUDA call is made."""
import ctypes
import os
import re

import pytest

import w8a8_smoothquant_gemm_b200 as sq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sq_w8a8.h")

INVALID, UNSUPPORTED, ALIGN, WORKSPACE = 1, 2, 3, 5
F32, BF16, I32 = 0, 1, 2


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", text)))


def test_header_declarations_are_exported():
    L = sq.lib()
    names = declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n


def test_library_has_no_cuda_runtime_or_driver_link_dependency():
    # the runtime is linked statically and the driver is reached through the runtime's
    # entry-point query, so the library loads on a machine without a GPU driver
    import subprocess
    out = subprocess.run(["ldd", sq.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcudart" not in out and "libcuda.so" not in out


def test_status_strings_and_version():
    L = sq.lib()
    assert L.sq_status_string(0) == b"SQ_OK"
    assert L.sq_status_string(5) == b"SQ_ERR_WORKSPACE"
    assert L.sq_abi_version() == 102


# fake, never dereferenced device addresses with chosen alignment
A16 = ctypes.c_void_p(0x10000)
A16b = ctypes.c_void_p(0x20000)
A16c = ctypes.c_void_p(0x30000)
A8 = ctypes.c_void_p(0x10008)
NULL = None


def test_calib_absmax_validation():
    f = sq.lib().sq_calib_absmax
    assert f(A16, BF16, 4, 64, 64, 2, 0, A16b, NULL) == INVALID        # bad axis
    assert f(A16, BF16, 4, 64, 64, 0, 3, A16b, NULL) == INVALID        # bad accumulate
    assert f(A16, I32, 4, 64, 64, 0, 0, A16b, NULL) == INVALID         # int32 input
    assert f(NULL, BF16, 4, 64, 64, 0, 0, A16b, NULL) == INVALID       # null x
    assert f(A16, BF16, 4, 64, 32, 0, 0, A16b, NULL) == INVALID        # ld < cols
    assert f(A16, BF16, -1, 64, 64, 0, 0, A16b, NULL) == INVALID       # negative rows
    assert f(A8, BF16, 4, 64, 64, 0, 0, A16b, NULL) == ALIGN           # misaligned x
    assert f(A16, BF16, 4, 60, 64, 0, 0, A16b, NULL) == ALIGN          # 120-byte rows
    assert f(A16, F32, 4, 64, 66, 0, 0, A16b, NULL) == ALIGN           # ld not 16 bytes
    assert f(A16, BF16, 4, 64, 64, 0, 0, NULL, NULL) == INVALID        # null out
    assert f(A16, BF16, 4, 0, 0, 0, 0, NULL, NULL) == 0                # nothing to do


def test_calib_ln_absmax_validation():
    f = sq.lib().sq_calib_ln_absmax
    assert f(A16, BF16, 4, 64, 64, NULL, NULL, 1e-5, 0, A16b, NULL) == INVALID     # null gamma
    assert f(A16, BF16, 4, 0, 0, A16c, NULL, 1e-5, 0, A16b, NULL) == INVALID       # K = 0
    assert f(A16, BF16, 4, 24, 24, A16c, NULL, 1e-5, 0, A16b, NULL) == ALIGN       # 48-byte rows, K % 16
    assert f(A16, BF16, 4, 65552, 65552, A16c, NULL, 1e-5, 0, A16b, NULL) == UNSUPPORTED
    assert f(A16, F32, 4, 32784, 32784, A16c, NULL, 1e-5, 0, A16b, NULL) == UNSUPPORTED
    assert f(A16, BF16, 4, 64, 64, A16c, NULL, -1.0, 0, A16b, NULL) == INVALID     # eps < 0


def test_smooth_factors_validation():
    f = sq.lib().sq_smooth_factors
    assert f(A16, A16b, 64, ctypes.c_float(1.5), A16c, NULL) == INVALID
    assert f(A16, A16b, 64, ctypes.c_float(-0.1), A16c, NULL) == INVALID
    assert f(A16, A16b, 64, ctypes.c_float(float("nan")), A16c, NULL) == INVALID
    assert f(NULL, A16b, 64, ctypes.c_float(0.5), A16c, NULL) == INVALID
    assert f(A16, A16b, -3, ctypes.c_float(0.5), A16c, NULL) == INVALID
    assert f(NULL, NULL, 0, ctypes.c_float(0.5), NULL, NULL) == 0


def test_fold_validation():
    f = sq.lib().sq_fold_quant_weights
    ok = dict(W=A16, dt=BF16, K=64, N=32, ldw=32, s=A16b, g=NULL, b=NULL, wq=A16c, sw=A16b, gf=NULL, bf=NULL)

    def call(**kw):
        a = {**ok, **kw}
        return f(a["W"], a["dt"], a["K"], a["N"], a["ldw"], a["s"], a["g"], a["b"], a["wq"], a["sw"], a["gf"],
                 a["bf"], NULL)

    assert call(s=NULL) == INVALID
    assert call(wq=NULL) == INVALID
    assert call(K=40, ldw=32) == ALIGN                     # K % 16 != 0
    assert call(wq=A8) == ALIGN
    assert call(N=36, ldw=36) == ALIGN                     # 72-byte rows
    assert call(K=0) == 0 and call(N=0, ldw=0) == 0


SQ_MAX_K_PLUS = 133152  # next multiple of 16 above the int32 accumulator bound


def test_fold_rejects_k_beyond_int32_range():
    f = sq.lib().sq_fold_quant_weights
    assert f(A16, BF16, SQ_MAX_K_PLUS, 32, 32, A16b, NULL, NULL, A16c, A16b, NULL, NULL, NULL) == UNSUPPORTED


def test_ln_smooth_quant_validation():
    f = sq.lib().sq_ln_smooth_quant
    # both modes / neither mode
    assert f(A16, BF16, 4, 64, 64, A16b, NULL, A16c, 1e-5, A16c, A16b, NULL) == INVALID
    assert f(A16, BF16, 4, 64, 64, NULL, NULL, NULL, 1e-5, A16c, A16b, NULL) == INVALID
    assert f(A16, BF16, 4, 64, 64, NULL, A16b, A16c, 1e-5, A16c, A16b, NULL) == INVALID   # beta without gamma
    assert f(A16, BF16, 4, 64, 64, A8, NULL, NULL, 1e-5, A16c, A16b, NULL) == ALIGN
    assert f(A16, BF16, 4, 40, 40, NULL, NULL, A16c, 1e-5, A16c, A16b, NULL) == ALIGN      # K % 16
    assert f(A16, BF16, 4, 64, 64, NULL, NULL, A16c, 1e-5, NULL, A16b, NULL) == INVALID    # null xq
    assert f(A16, BF16, 4, 65552, 65552, NULL, NULL, A16c, 1e-5, A16c, A16b, NULL) == UNSUPPORTED
    assert f(A16, BF16, 0, 64, 64, NULL, NULL, A16c, 1e-5, NULL, NULL, NULL) == 0          # M = 0


def test_gemm_validation():
    f = sq.lib().sq_w8a8_gemm

    def call(xq=A16, sx=A16b, wq=A16c, sw=A16b, M=8, N=32, K=64, y=A16, ydt=BF16, ldy=32, ws=NULL, wsb=0):
        return f(xq, sx, wq, sw, M, N, K, y, ydt, ldy, ws, wsb, NULL)

    assert call(K=0) == INVALID
    assert call(ydt=7) == INVALID
    assert call(ldy=16) == INVALID
    assert call(xq=NULL) == INVALID
    assert call(sx=NULL) == INVALID                 # scales needed for bf16 output
    assert call(K=40) == ALIGN
    assert call(wq=A8) == ALIGN
    assert call(y=ctypes.c_void_p(0x10001)) == ALIGN  # output not aligned to its element
    assert call(ws=ctypes.c_void_p(0x10010)) == ALIGN
    assert call(K=SQ_MAX_K_PLUS) == UNSUPPORTED
    assert call(M=0) == 0 and call(N=0, ldy=0) == 0


def test_gemm_noalloc_checks_arguments_before_its_scratch_size():
    """The no-allocation GEMM reports a bad argument as sq_w8a8_gemm does, even for a shape whose
    workspace would not fit its built-in scratch (which is checked only after the arguments)."""
    f = sq.lib().sq_w8a8_gemm_noalloc
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f.argtypes = [P, P, P, P, I64, I64, I64, P, I, I64, P]
    f.restype = I

    def call(xq=A16, sx=A16b, wq=A16c, sw=A16b, M=96, N=1 << 20, K=65536, y=A16, ydt=BF16, ldy=1 << 20):
        return f(xq, sx, wq, sw, M, N, K, y, ydt, ldy, NULL)

    assert call(xq=NULL) == INVALID
    assert call(sx=NULL) == INVALID
    assert call(K=40) == ALIGN
    assert call(y=ctypes.c_void_p(0x10001)) == ALIGN
    assert call(K=SQ_MAX_K_PLUS) == UNSUPPORTED
    assert call(ldy=16) == INVALID
    assert call(M=0) == 0


def test_gemm_rowmax_and_codes_validation():
    g = sq.lib().sq_w8a8_gemm_rowmax

    def call(xq=A16, sx=A16b, wq=A16c, sw=A16b, M=8, N=32, K=64, y=A16, ydt=BF16, ldy=32, rmax=A16b, ws=NULL, wsb=0):
        return g(xq, sx, wq, sw, M, N, K, y, ydt, ldy, rmax, ws, wsb, NULL)

    assert call(ydt=I32) == INVALID          # the row max needs scaled outputs
    assert call(rmax=NULL) == INVALID
    assert call(rmax=ctypes.c_void_p(0x10002)) == INVALID
    assert call(xq=NULL) == INVALID
    assert call(K=40) == ALIGN
    assert call(M=0) == 0
    c = sq.lib().sq_quant_codes
    assert c(A16, BF16, 4, 64, 64, NULL, A16b, A16c, NULL) == INVALID       # null rowmax
    assert c(A16, BF16, 4, 0, 0, A16b, A16b, A16c, NULL) == INVALID         # K = 0
    assert c(A16, BF16, 4, 24, 24, A16b, A16b, A16c, NULL) == ALIGN         # 48-byte rows
    assert c(A16, BF16, 4, 64, 64, A16b, A8, A16c, NULL) == ALIGN           # misaligned codes
    assert c(A16, I32, 4, 64, 64, A16b, A16b, A16c, NULL) == INVALID        # int32 input
    assert c(A16, BF16, 0, 64, 64, NULL, NULL, NULL, NULL) == 0             # nothing to do


def test_wait_limit_symbol():
    f = sq.lib().sq_set_wait_limit
    assert f.argtypes[0] is ctypes.c_uint64


def test_workspace_size_validation():
    f = sq.lib().sq_w8a8_gemm_workspace_size
    assert f(4, 4, 0) == ctypes.c_size_t(-1).value
    assert f(4, 4, 24) == ctypes.c_size_t(-1).value
    assert f(0, 64, 64) == 0


def test_device_error_null_pointer():
    assert sq.lib().sq_device_error(NULL, 0, NULL) == INVALID


def test_ln_smooth_quant_per_tensor_validation():
    f = sq.lib().sq_ln_smooth_quant_per_tensor
    ok = (A16, BF16, 4, 64, 64, NULL, NULL, A16c, 1e-5, 0, A16b, A16c, A16b, NULL)
    args = list(ok)
    args[10] = NULL
    assert f(*args) == INVALID                       # no scale
    args = list(ok)
    args[9] = 2
    assert f(*args) == INVALID                       # static flag not 0/1
    args = list(ok)
    args[5] = A16b
    assert f(*args) == INVALID                       # both modes
    args = list(ok)
    args[3] = 40
    args[4] = 40
    assert f(*args) == ALIGN                         # K % 16
    args = list(ok)
    args[2] = 0
    assert f(*args) == 0                             # M = 0: nothing to do


def test_alpha_search_validation():
    L = sq.lib()
    f = L.sq_alpha_search
    ws_need = L.sq_alpha_search_workspace_size(64, 256, 128)
    assert 0 < ws_need < (1 << 40)
    assert L.sq_alpha_search_workspace_size(64, 250, 128) == (1 << 64) - 1   # K % 16 != 0
    a = (ctypes.c_float * 3)(0.0, 0.5, 1.0)
    bad = (ctypes.c_float * 2)(0.5, 1.5)
    W = ctypes.c_void_p(0x40000)
    ws = ctypes.c_void_p(0x100000)
    err = ctypes.c_void_p(0x50000)
    ok = (A16, BF16, 64, 256, 256, A16b, NULL, ctypes.c_float(1e-5), W, BF16, 128, 128)
    assert f(*ok, a, 0, err, ws, ws_need, NULL) == INVALID                  # no strengths
    assert f(*ok, a, 257, err, ws, ws_need, NULL) == INVALID                # too many
    assert f(*ok, bad, 2, err, ws, ws_need, NULL) == INVALID                # alpha > 1
    assert f(*ok, a, 3, NULL, ws, ws_need, NULL) == INVALID                 # no output
    assert f(*ok, a, 3, err, ws, ws_need - 1, NULL) == WORKSPACE            # workspace too small
    assert f(*ok, a, 3, err, ctypes.c_void_p(0x100010), ws_need, NULL) == ALIGN
    assert f(A16, BF16, 64, 256, 256, NULL, A16c, ctypes.c_float(1e-5), W, BF16, 128, 128,
             a, 3, err, ws, ws_need, NULL) == INVALID                       # beta without gamma


def test_fold_kernel_launches_routing():
    f = sq.lib().sq_fold_kernel_launches
    assert f(A16, BF16, 0, 64, 64) == 0
    assert f(A16, BF16, 4096, 4096, 4096) == 1             # one-pass cluster fold
    assert f(A16, BF16, 4096, 28672, 28672) == 3           # streaming two-pass fold
    assert f(A16, BF16, 49152, 64, 64) == 3                # cluster block too tall
    assert f(A8, BF16, 49152, 64, 64) == 1                 # unaligned: strip kernel
    assert f(A16, F32, 4096, 28672, 28672) == 1            # fp32 weights: strip kernel


def test_workspace_sizes_follow_the_launch_plan():
    """Host-only launch planning (148 SMs when no device answers, as on a B200): the workspace
    each GEMM shape asks for, derived by hand from the planning rules."""
    ws = sq.sq_w8a8_gemm_workspace_size
    # swap-AB decode, 32 weight tiles on 148 SMs: stream-K over all 148 CTAs; the larger of the
    # tile sums (32 tiles) and two partial slots per CTA (296), of 128 x BN int32 (BN = 16)
    assert ws(1, 4096, 4096) == 296 * 128 * 16 * 4
    # 224 tiles: one full wave of whole tiles, then 76 tiles stream-K over 148 CTAs
    assert ws(16, 28672, 4096) == 296 * 128 * 16 * 4
    # BN = 64 for 33-64 tokens
    assert ws(64, 4096, 14336) == 296 * 128 * 64 * 4
    # CTA pairs, 36 tiles on 74 pairs: K split 2 ways, [2][M][N] int32
    assert ws(1536, 1536, 4096) == 2 * 1536 * 1536 * 4
    # CTA pairs, 384 tiles = 5 waves of 74 + 14, K = 384 blocks: the 14 tail tiles in 5 pieces
    # of 77 blocks, [5][14][256][256] int32
    assert ws(2048, 12288, 49152) == 5 * 14 * 256 * 256 * 4
    # the same tiling with K = 96 blocks: pieces would be shorter than 64 blocks, no split tail
    assert ws(2048, 12288, 12288) == 0
    # 76 tiles = 74 + 2, K = 129 blocks: 2 pieces (65 + 64 blocks) per tail tile
    assert ws(300, 9572, 16400) == 2 * 2 * 256 * 256 * 4
    # 768 tiles = 10 waves + 28, K = 32 blocks: no split tail
    assert ws(8192, 6144, 4096) == 0


def test_binding_has_no_fallback(monkeypatch):
    """Without the library every call raises; host tensors are refused, not computed on the CPU."""
    import torch
    x = torch.zeros(2, 16)
    with pytest.raises(ValueError):
        sq.sq_ln_smooth_quant(x, s=torch.ones(16))
    monkeypatch.setattr(sq, "_lib", None)
    monkeypatch.setattr(sq, "LIB_PATH", os.path.join(ROOT, "w8a8_smoothquant_gemm_b200", "no_such_library.so"))
    with pytest.raises(OSError):
        sq.lib()

"""sq_w8a8_gemm_noalloc: the GEMM entry point for callers that cannot allocate device memory
(a plug-in inside a host program that owns all device memory through its own pool, or a
latency-critical loop where cudaMalloc may synchronise the device).  It keeps its split-K
partial sums in a scratch array compiled into the library instead of a caller-provided
workspace.  These tests call it through the C ABI and compare it with sq_w8a8_gemm (which
gets a workspace from torch), on two calls in a row so that the scratch's leftover contents
from the first call cannot change the second result.  The file is named to be collected
last; it passes alone in a fresh process and after the other tests."""
import ctypes
import os
import re

import numpy as np
import pytest
import torch

import w8a8_smoothquant_gemm_b200 as sq

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sq_w8a8.h")


def scratch_bytes() -> int:
    m = re.search(r"#define\s+SQ_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", open(HEADER).read())
    return int(m.group(1)) << int(m.group(2))


def noalloc_fn():
    f = sq.lib().sq_w8a8_gemm_noalloc
    P, I64, I = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    f.argtypes = [P, P, P, P, I64, I64, I64, P, I, I64, P]
    f.restype = I
    return f


def call_noalloc(xq, sx, wq, sw, y):
    M, K = xq.shape
    N = wq.shape[0]
    ydt = {torch.bfloat16: sq.SQ_BF16, torch.float32: sq.SQ_F32, torch.int32: sq.SQ_I32}[y.dtype]
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())  # noqa: E731
    return noalloc_fn()(ptr(xq), ptr(sx), ptr(wq), ptr(sw), M, N, K, ptr(y), ydt, y.stride(0),
                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def bf16_close(a: torch.Tensor, b: torch.Tensor) -> bool:
    """Within 1 bf16 ulp or 4e-3 relative, the tolerance of the GPU parity tests."""
    a64, b64 = a.double().cpu().numpy(), b.double().cpu().numpy()
    ulp = np.spacing(np.abs(b64).astype(np.float32)).astype(np.float64) * 65536.0
    d = np.abs(a64 - b64)
    return bool(np.all((d <= ulp) | (d <= 4e-3 * np.abs(b64))))


def inputs(M, N, K, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(seed)
    xq = torch.randint(-127, 128, (M, K), generator=g, device=DEV, dtype=torch.int32).to(torch.int8)
    wq = torch.randint(-127, 128, (N, K), generator=g, device=DEV, dtype=torch.int32).to(torch.int8)
    sx = torch.rand(M, generator=g, device=DEV) * 0.5 + 1e-3
    sw = torch.rand(N, generator=g, device=DEV) * 1e-2 + 1e-5
    return xq, sx, wq, sw


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (64, 6144, 4096), (3, 1000, 14336), (200, 512, 1024),
                                   (1, 28672, 4096)])
def test_noalloc_matches_workspace_gemm_on_two_calls(M, N, K):
    need = sq.sq_w8a8_gemm_workspace_size(M, N, K)
    if not 0 < need <= scratch_bytes():
        pytest.skip(f"on this device the launch for {M}x{N}x{K} needs {need} bytes of scratch (premise: 0 < need "
                    f"<= {scratch_bytes()})")
    xq, sx, wq, sw = inputs(M, N, K, M + N + K)
    ref_y = sq.sq_w8a8_gemm(xq, sx, wq, sw)
    ref_acc = sq.sq_w8a8_gemm(xq, None, wq, None, out_dtype=torch.int32)
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
        acc = torch.zeros(M, N, dtype=torch.int32, device=DEV)
        assert call_noalloc(xq, sx, wq, sw, y) == 0
        assert call_noalloc(xq, None, wq, None, acc) == 0
        torch.cuda.synchronize()
        assert bf16_close(y, ref_y)
        assert torch.equal(acc, ref_acc)
    assert sq.sq_device_error(clear=True) == 0


def test_noalloc_without_split_and_after_a_different_shape():
    # a shape that does not split K uses no scratch; run it between two split shapes
    for M, N, K in ((16, 4096, 4096), (4096, 1024, 512), (64, 4096, 14336)):
        xq, sx, wq, sw = inputs(M, N, K, 7 * M + K)
        y = torch.empty(M, N, dtype=torch.bfloat16, device=DEV)
        assert call_noalloc(xq, sx, wq, sw, y) == 0
        assert bf16_close(y, sq.sq_w8a8_gemm(xq, sx, wq, sw))


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # the first candidate whose launch on this device needs more scratch than the array holds
    candidates = [(1536, 1536, 4096), (128, 5120, 4096), (2048, 2048, 8192), (4096, 4096, 4096)]
    big = [c for c in candidates if sq.sq_w8a8_gemm_workspace_size(*c) > scratch_bytes()]
    if not big:
        pytest.skip("no candidate shape needs more than the built-in scratch on this device")
    M, N, K = big[0]
    xq, sx, wq, sw = inputs(M, N, K, 3)
    y = torch.zeros(M, N, dtype=torch.bfloat16, device=DEV)
    assert call_noalloc(xq, sx, wq, sw, y) == 5  # SQ_ERR_WORKSPACE, nothing launched
    torch.cuda.synchronize()
    assert not y.any()

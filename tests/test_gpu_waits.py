"""Failure detection without a GPU fault: every bounded wait in the kernels runs out at once
(sq_set_wait_limit(0), a diagnostic of the library), and each kernel that waits -- the GEMM, the
staged activation-row kernel, the cluster fold and the streaming fold -- must return promptly,
report its bit in the device error word, and leave a usable context: the same call with the
default limit then matches the oracle again.  No wait is made to fail by a fault, a trap or a
hang: the limit runs out before the kernel looks at its barrier."""
import time

import numpy as np
import pytest
import torch

import oracle as O
import sq_inputs
import w8a8_smoothquant_gemm_b200 as sq

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
GEMM_BITS, FOLD_BIT, ROW_BIT = 0x7, 0x8, 0x10


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    return t.view(torch.int16).numpy().view(np.uint16) if t.dtype == torch.bfloat16 else t.numpy()


@pytest.fixture
def waits_run_out():
    """Every wait runs out at once while the test body runs; the default limit comes back even
    if the body fails."""
    torch.cuda.synchronize()
    sq.sq_device_error(clear=True)
    sq.sq_set_wait_limit(0)
    try:
        yield
    finally:
        torch.cuda.synchronize()
        sq.sq_set_wait_limit(sq.WAIT_LIMIT_DEFAULT_NS)
        sq.sq_device_error(clear=True)


def timed(fn):
    t0 = time.perf_counter()
    fn()
    torch.cuda.synchronize()
    return time.perf_counter() - t0


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (1, 28672, 4096), (2048, 1024, 2048)])
def test_gemm_gives_up(waits_run_out, M, N, K):
    rng = np.random.default_rng(1)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    dx, dw = dev(xq), dev(wq)
    assert timed(lambda: sq.sq_w8a8_gemm(dx, None, dw, None, out_dtype=torch.int32)) < 5.0
    assert sq.sq_device_error(clear=True) & GEMM_BITS
    sq.sq_set_wait_limit(sq.WAIT_LIMIT_DEFAULT_NS)
    acc = sq.sq_w8a8_gemm(dx, None, dw, None, out_dtype=torch.int32)
    assert np.array_equal(host(acc), O.w8a8_gemm(xq, None, wq, None, "i32"))
    assert sq.sq_device_error(clear=True) == 0


@pytest.mark.parametrize("mode", ["ln", "plain", "calib"])
def test_row_kernel_gives_up(waits_run_out, mode):
    # few rows of a model width: the staged row kernel (bulk copies into a shared-memory ring)
    c = sq_inputs.make_case(16, 4096, 8, 3, beta_std=0.05)
    x, g = dev(c.x), dev(c.gamma)
    s = np.exp(np.random.default_rng(2).uniform(-1, 2, 4096)).astype(np.float32)

    def call():
        if mode == "ln":
            return sq.sq_ln_smooth_quant(x, gamma_f=g)
        if mode == "plain":
            return sq.sq_ln_smooth_quant(x, s=dev(s))
        return sq.sq_calib_ln_absmax(x, g)

    assert timed(call) < 5.0
    assert sq.sq_device_error(clear=True) & ROW_BIT
    sq.sq_set_wait_limit(sq.WAIT_LIMIT_DEFAULT_NS)
    out = call()
    if mode == "ln":
        r_xq, r_sx = O.ln_smooth_quant(c.x, gamma_f=c.gamma)
        assert np.array_equal(host(out[0]), r_xq) and np.array_equal(host(out[1]), r_sx)
    elif mode == "plain":
        r_xq, r_sx = O.ln_smooth_quant(c.x, s=s)
        assert np.array_equal(host(out[0]), r_xq) and np.array_equal(host(out[1]), r_sx)
    else:
        assert np.array_equal(host(out), O.calib_ln_absmax(c.x, c.gamma))
    assert sq.sq_device_error(clear=True) == 0


@pytest.mark.parametrize("K,N,launches", [(4096, 4096, 1), (4096, 28672, 3)])
def test_fold_gives_up(waits_run_out, K, N, launches):
    _, W, g, _ = sq_inputs.torch_case(1, K, N, 9, DEV)
    assert sq.sq_fold_kernel_launches(W) == launches  # the cluster fold, then the streaming fold
    s = np.exp(np.random.default_rng(K).uniform(-1, 2, K)).astype(np.float32)
    assert timed(lambda: sq.sq_fold_quant_weights(W, dev(s), g)) < 5.0
    assert sq.sq_device_error(clear=True) & FOLD_BIT
    sq.sq_set_wait_limit(sq.WAIT_LIMIT_DEFAULT_NS)
    wq, sw, gf, _ = sq.sq_fold_quant_weights(W, dev(s), g)
    r_wq, r_sw, r_gf, _ = O.fold_quant_weights(host(W), s, host(g))
    assert np.array_equal(host(sw), r_sw) and np.array_equal(host(wq), r_wq) and np.array_equal(host(gf), r_gf)
    assert sq.sq_device_error(clear=True) == 0

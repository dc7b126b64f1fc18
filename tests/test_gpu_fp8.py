"""GPU parity of the FP8 (E4M3) variant against the CPU oracle on the same seeded bytes.

Codes and scales are compared bit for bit (both sides take the code decision as E4M3 of the
correctly rounded binary32 quotient).  The GEMM accumulates exact E4M3 products in binary32
on the tensor cores, in the hardware's order, so its accumulator is checked against the
oracle's exact sum within the binary32 summation bound |acc - exact| <= K * 2^-23 * sum|p|
(any order of K rounded additions; 2^-23 also covers truncating adders), and the bf16
output within that error plus one bf16 ulp."""
import numpy as np
import pytest
import torch

import oracle as O
import sq_inputs
import w8a8_smoothquant_gemm_b200 as sq

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


@pytest.fixture(autouse=True)
def _no_device_error():
    sq.sq_device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert sq.sq_device_error(clear=True) == 0


# ----------------------------------------------------------------------------- fold
@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("K,N", [(16, 8), (256, 200), (4096, 4096), (1040, 3000), (14336, 512), (49152, 64),
                                 (40016, 1288)])
def test_fold_fp8(dt, K, N):
    if dt == "f32" and K > 4096:
        pytest.skip("fp32 weights are covered by the smaller shapes")
    c = sq_inputs.make_case(2, K, N, K + N, x_dtype=dt, w_dtype=dt)
    s = np.exp(np.random.default_rng(K).uniform(-1, 1.5, K)).astype(np.float32)
    W = c.W.copy()
    W[:, 3] = 0                                               # zero column: scale 0, codes +0
    if dt == "bf16":
        W[::7, 5] = np.uint16(0x8000)                         # -0 entries
    wq, sw, gf, _ = sq.sq_fold_quant_weights_fp8(dev(W), dev(s), dev(c.gamma))
    r_wq, r_sw, r_gf, _ = O.fold_quant_weights_fp8(W, s, c.gamma)
    assert np.array_equal(host(sw), r_sw)
    assert np.array_equal(host(wq), r_wq)
    assert np.array_equal(host(gf), r_gf)


def test_fold_fp8_streaming_padded():
    """E4M3 codes on the streaming two-pass route with a padded leading dimension (ragged last
    row tile and column strip, a zero column, -0 entries)."""
    K, N, extra = 40016, 1288, 8
    _, W, g, _ = sq_inputs.torch_case(1, K, N, 13, DEV, w_std=0.015)
    W = torch.nn.functional.pad(W, (0, extra))[:, :N]
    W[:, 3] = 0
    W[::5, 6] = -0.0
    assert sq.sq_fold_kernel_launches(W) == 3
    s = np.exp(np.random.default_rng(K).uniform(-1, 1.5, K)).astype(np.float32)
    wq, sw, gf, _ = sq.sq_fold_quant_weights_fp8(W, dev(s), g)
    r_wq, r_sw, r_gf, _ = O.fold_quant_weights_fp8(host(W), s, host(g))
    assert np.array_equal(host(sw), r_sw)
    assert np.array_equal(host(wq), r_wq)
    assert np.array_equal(host(gf), r_gf)


# ----------------------------------------------------------------------------- per-token quantiser
@pytest.mark.parametrize("M,K", [(1, 16), (5, 256), (33, 2048), (64, 4096), (3, 16400), (2, 49152),
                                 (1031, 4096), (1029, 14336), (1030, 512), (1030, 12288), (1100, 8192)])
@pytest.mark.parametrize("mode", ["ln", "plain"])
def test_ln_smooth_quant_fp8(M, K, mode):
    c = sq_inputs.make_case(M, K, 8, 3 * M + K, beta_std=0.05)
    s = np.exp(np.random.default_rng(K + 3).uniform(-1, 3, K)).astype(np.float32)
    x = c.x.copy()
    if M > 2:
        x[1] = 0                                              # zero row
        x[2, ::3] = np.uint16(0x8000)                         # -0 inputs keep their sign in plain mode
    if mode == "ln":
        gf, bf = (c.gamma / s).astype(np.float32), (c.beta / s).astype(np.float32)
        xq, sx = sq.sq_ln_smooth_quant_fp8(dev(x), gamma_f=dev(gf), beta_f=dev(bf))
        r_xq, r_sx = O.ln_smooth_quant_fp8(x, gamma_f=gf, beta_f=bf)
    else:
        xq, sx = sq.sq_ln_smooth_quant_fp8(dev(x), s=dev(s))
        r_xq, r_sx = O.ln_smooth_quant_fp8(x, s=s)
        if M > 2:
            assert (r_xq[2] == 0x80).any()
    assert np.array_equal(host(sx), r_sx)
    assert np.array_equal(host(xq), r_xq)


# ----------------------------------------------------------------------------- GEMM
def _finite_codes(rng, shape):
    fin = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    return rng.choice(fin, shape).astype(np.uint8)


def _acc_bound(xq, wq):
    ax = np.abs(O.e4m3_decode(xq).astype(np.float64))
    aw = np.abs(O.e4m3_decode(wq).astype(np.float64))
    K = xq.shape[1]
    return K * 2.0 ** -23 * (ax @ aw.T)


GEMM_SHAPES = [(1, 8, 16), (1, 200, 272), (7, 24, 32), (16, 256, 256), (16, 4096, 4096), (64, 130, 1024),
               (100, 1000, 512), (129, 264, 128), (256, 512, 4096), (300, 1024, 1040), (2048, 512, 96),
               (5, 1000, 8192), (7, 5120, 2048), (1, 19072, 272), (16, 28672, 1024), (3, 4096, 14336),
               (2048, 12200, 128)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_fp8_accumulator(M, N, K):
    rng = np.random.default_rng(M * 7 + N + K)
    xq, wq = _finite_codes(rng, (M, K)), _finite_codes(rng, (N, K))
    ones_m, ones_n = np.ones(M, np.float32), np.ones(N, np.float32)
    got = host(sq.sq_w8a8_gemm_fp8(dev(xq), dev(ones_m), dev(wq), dev(ones_n), out_dtype=torch.float32))
    exact, _ = O.fp8_gemm(xq, ones_m, wq, ones_n, "f32")
    err = np.abs(got.astype(np.float64) - exact)
    assert np.all(err <= _acc_bound(xq, wq)), float(np.max(err / np.maximum(_acc_bound(xq, wq), 1e-300)))


def test_gemm_fp8_split_tail_sampled_rows():
    """CTA-pair tiles in a full wave plus two tiles split along K over the idle pairs (300 x
    9572 x 16400): the pieces' fp32 partials are summed in split order; sampled rows, every
    column, within the bound."""
    M, N, K = 300, 9572, 16400
    rng = np.random.default_rng(41)
    xq, wq = _finite_codes(rng, (M, K)), _finite_codes(rng, (N, K))
    ones_m, ones_n = np.ones(M, np.float32), np.ones(N, np.float32)
    ws = torch.zeros(sq.sq_w8a8_gemm_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
    got = host(sq.sq_w8a8_gemm_fp8(dev(xq), dev(ones_m), dev(wq), dev(ones_n), out_dtype=torch.float32,
                                   workspace=ws))
    assert not ws.any()
    r = np.array([0, 1, 128, 255, 256, 299])
    exact, _ = O.fp8_gemm(xq[r], ones_m[r], wq, ones_n, "f32")
    err = np.abs(got[r].astype(np.float64) - exact)
    assert np.all(err <= _acc_bound(xq[r], wq))


def test_gemm_fp8_and_int8_share_a_workspace():
    """FP8 and INT8 GEMMs of split shapes take turns on one zero-filled workspace: every result
    holds (FP8 within its bound, and the same bits on a repeated call; INT8 exact) and the
    workspace is all zero after each call."""
    shapes = [(16, 4096, 4096), (1, 28672, 4096), (300, 1024, 1040), (64, 6144, 4096)]
    ws = torch.zeros(max(sq.sq_w8a8_gemm_workspace_size(*sh) for sh in shapes), dtype=torch.uint8, device=DEV)
    rng = np.random.default_rng(21)
    for M, N, K in shapes:
        xq, wq = _finite_codes(rng, (M, K)), _finite_codes(rng, (N, K))
        ones_m, ones_n = np.ones(M, np.float32), np.ones(N, np.float32)
        a = sq.sq_w8a8_gemm_fp8(dev(xq), dev(ones_m), dev(wq), dev(ones_n), out_dtype=torch.float32, workspace=ws)
        assert not ws.any()
        b = sq.sq_w8a8_gemm_fp8(dev(xq), dev(ones_m), dev(wq), dev(ones_n), out_dtype=torch.float32, workspace=ws)
        assert not ws.any()
        exact, _ = O.fp8_gemm(xq, ones_m, wq, ones_n, "f32")
        assert np.all(np.abs(host(a).astype(np.float64) - exact) <= _acc_bound(xq, wq))
        assert np.array_equal(host(a), host(b))  # a fixed order of additions: reproducible
        iq = rng.integers(-127, 128, (M, K)).astype(np.int8)
        iw = rng.integers(-127, 128, (N, K)).astype(np.int8)
        acc = sq.sq_w8a8_gemm(dev(iq), None, dev(iw), None, out_dtype=torch.int32, workspace=ws)
        assert not ws.any()
        assert np.array_equal(host(acc), O.w8a8_gemm(iq, None, iw, None, "i32"))


@pytest.mark.parametrize("M,N,K", [(16, 4096, 4096), (300, 1024, 1040), (2048, 512, 96)])
def test_gemm_fp8_bf16_epilogue(M, N, K):
    rng = np.random.default_rng(M + N + K)
    xq, wq = _finite_codes(rng, (M, K)), _finite_codes(rng, (N, K))
    sx = np.exp(rng.uniform(-8, 0, M)).astype(np.float32)
    sw = np.exp(rng.uniform(-8, 0, N)).astype(np.float32)
    y = host(sq.sq_w8a8_gemm_fp8(dev(xq), dev(sx), dev(wq), dev(sw)))
    exact, ref = O.fp8_gemm(xq, sx, wq, sw, "bf16")
    g = O.bf16_to_f32(y).astype(np.float64)
    r = O.bf16_to_f32(ref).astype(np.float64)
    ulp = np.spacing(np.abs(r).astype(np.float32)).astype(np.float64) * 65536.0
    slack = _acc_bound(xq, wq) * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64) * (1 + 2.0 ** -20)
    assert np.all(np.abs(g - r) <= ulp + slack)


def test_fp8_linear_end_to_end():
    """Calibration, smoothing, FP8 fold, FP8 quantiser and FP8 GEMM against the oracle's path."""
    M, K, N = 1100, 4096, 768
    x, W, gamma, _ = sq_inputs.torch_case(M, K, N, 41, DEV, w_std=0.02)
    ax = sq.sq_calib_ln_absmax(x, gamma)
    aw = sq.sq_calib_absmax(W, 1)
    s = sq.sq_smooth_factors(ax, aw, 0.5)
    wq, sw, gf, _ = sq.sq_fold_quant_weights_fp8(W, s, gamma)
    xq, sx = sq.sq_ln_smooth_quant_fp8(x, gamma_f=gf)
    y = sq.sq_w8a8_gemm_fp8(xq, sx, wq, sw)
    hx, hW, hs = host(x), host(W), host(s)
    r_wq, r_sw, r_gf, _ = O.fold_quant_weights_fp8(hW, hs, host(gamma))
    assert np.array_equal(host(wq), r_wq) and np.array_equal(host(sw), r_sw)
    r_xq, r_sx = O.ln_smooth_quant_fp8(hx, gamma_f=r_gf)
    assert np.array_equal(host(xq), r_xq) and np.array_equal(host(sx), r_sx)
    rows = np.linspace(0, M - 1, 7).astype(int)
    exact, ref = O.fp8_gemm(r_xq[rows], r_sx[rows], r_wq, r_sw, "bf16")
    g = O.bf16_to_f32(host(y)[rows]).astype(np.float64)
    r = O.bf16_to_f32(ref).astype(np.float64)
    ulp = np.spacing(np.abs(r).astype(np.float32)).astype(np.float64) * 65536.0
    slack = _acc_bound(r_xq[rows], r_wq) * r_sx[rows, None].astype(np.float64) * r_sw[None, :].astype(np.float64)
    assert np.all(np.abs(g - r) <= ulp + slack * (1 + 2.0 ** -20))
    # and the layer is close to the unquantised one
    Y = O.layernorm(hx[rows], host(gamma)).astype(np.float64) @ O.bf16_to_f32(hW).astype(np.float64)
    assert np.linalg.norm(g - Y) / np.linalg.norm(Y) < 0.08

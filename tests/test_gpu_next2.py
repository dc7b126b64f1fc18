"""The next linear's quantiser fused into the previous GEMM ("4.2 W8A8 量化与 SmoothQuant",
sec. 6: a linear's input comes from a LayerNorm or from the previous GEMM's output, and the
smoothing folds into that previous layer; "量化：只压权重，与训练后量化（PTQ）", SmoothQuant
section: diag(s)^-1 folds offline into the preceding layer).

sq_w8a8_gemm_rowmax stores y like sq_w8a8_gemm and also the per-row max |y| of the stored values;
sq_quant_codes then quantises y per token from those maxima in one read.  Everything is compared
with the oracle bit for bit: the row maxima with the oracle's row absmax of the stored outputs,
the codes and scales with the oracle's per-token quantiser (plain mode, unit factors), and a
two-linear chain with the oracle's chain."""
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


# every launch route of the GEMM: decode whole tiles, stream-K with the reduction kernel, the
# CTA-pair tiles, and the pair tiles with split K
ROUTES = [(16, 36864, 256), (1, 4096, 4096), (64, 28672, 1024), (7, 1000, 8192), (300, 1024, 1040),
          (2048, 4096, 512), (256, 512, 4096)]


@pytest.mark.parametrize("M,N,K", ROUTES)
@pytest.mark.parametrize("out", ["bf16", "f32"])
def test_gemm_rowmax(M, N, K, out):
    rng = np.random.default_rng(M + N + K)
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 0.5, M).astype(np.float32)
    sw = rng.uniform(1e-5, 1e-2, N).astype(np.float32)
    if M > 2:
        xq[2] = 0  # a zero row: max 0
    odt = torch.bfloat16 if out == "bf16" else torch.float32
    y, rmax = sq.sq_w8a8_gemm_rowmax(dev(xq), dev(sx), dev(wq), dev(sw), out_dtype=odt)
    ref = O.w8a8_gemm(xq, sx, wq, sw, out)
    assert np.array_equal(host(y), ref)
    assert np.array_equal(host(rmax), O.calib_absmax(ref, 1))
    # a second call overwrites the maxima (no running max across calls)
    y2, rmax2 = sq.sq_w8a8_gemm_rowmax(dev(xq), dev(sx * np.float32(0.5)), dev(wq), dev(sw), out_dtype=odt, rowmax=rmax)
    assert np.array_equal(host(rmax2), O.calib_absmax(O.w8a8_gemm(xq, sx * np.float32(0.5), wq, sw, out), 1))


@pytest.mark.parametrize("M,K,dt", [(1, 16, "bf16"), (33, 4096, "bf16"), (2051, 12288, "bf16"), (5, 49152, "bf16"),
                                    (3, 98304, "bf16"), (300, 1040, "f32"), (70000, 32, "bf16")])
def test_quant_codes_match_the_per_token_quantiser(M, K, dt):
    c = sq_inputs.make_case(M, K, 8, M + K, x_dtype=dt)
    if M > 1:
        c.x[1] = 0  # an all-zero row: scale 0, zero codes
    rowmax = O.calib_absmax(c.x, 1)
    xq, sx = sq.sq_quant_codes(dev(c.x), dev(rowmax))
    r_xq, r_sx = O.ln_smooth_quant(c.x, s=np.ones(K, np.float32))
    assert np.array_equal(host(sx), r_sx)
    assert np.array_equal(host(xq), r_xq)


def test_two_linears_with_the_next_quantiser_fused_into_the_previous_gemm():
    """Linear A (LayerNorm in front) feeds linear B.  B's smoothing is folded into A's output
    scales; A's GEMM stores B's smoothed input in bf16 with its row maxima; B's codes come from
    those maxima in one pass; B's GEMM runs on them.  Every intermediate equals the oracle's chain,
    and the fused path equals the unfused one (GEMM, then the full per-token quantiser)."""
    M, K1, K2, N = 1029, 1024, 4096, 512
    c = sq_inputs.make_case(M, K1, K2, 31, beta_std=0.05)
    WB = sq_inputs.make_case(1, K2, N, 32).W
    x, WA, g, b, WBd = dev(c.x), dev(c.W), dev(c.gamma), dev(c.beta), dev(WB)
    sA = sq.sq_smooth_factors(sq.sq_calib_ln_absmax(x, g, b), sq.sq_calib_absmax(WA, 1), 0.5)
    wqA, swA, gfA, bfA = sq.sq_fold_quant_weights(WA, sA, g, b)
    xqA, sxA = sq.sq_ln_smooth_quant(x, gamma_f=gfA, beta_f=bfA)
    yA = sq.sq_w8a8_gemm(xqA, sxA, wqA, swA)  # calibration of B on A's output
    sB = sq.sq_smooth_factors(sq.sq_calib_absmax(yA, 0), sq.sq_calib_absmax(WBd, 1), 0.5)
    wqB, swB, _, _ = sq.sq_fold_quant_weights(WBd, sB)
    swA2 = sq.sq_fold_next_smoothing(swA, sB)
    # fused: A's GEMM emits y / s_B and its row maxima; B's codes in one pass
    yA2, rmax = sq.sq_w8a8_gemm_rowmax(xqA, sxA, wqA, swA2)
    xqB, sxB = sq.sq_quant_codes(yA2, rmax)
    yB = sq.sq_w8a8_gemm(xqB, sxB, wqB, swB)
    # unfused: the full quantiser with unit factors on the same stored output
    xqB_u, sxB_u = sq.sq_ln_smooth_quant(yA2, s=torch.ones(K2, dtype=torch.float32, device=DEV))
    assert torch.equal(xqB, xqB_u) and torch.equal(sxB, sxB_u)

    r_sA = O.smooth_factors(O.calib_ln_absmax(c.x, c.gamma, c.beta), O.calib_absmax(c.W, 1), 0.5)
    r_wqA, r_swA, r_gfA, r_bfA = O.fold_quant_weights(c.W, r_sA, c.gamma, c.beta)
    r_xqA, r_sxA = O.ln_smooth_quant(c.x, gamma_f=r_gfA, beta_f=r_bfA)
    r_yA = O.w8a8_gemm(r_xqA, r_sxA, r_wqA, r_swA, "bf16")
    r_sB = O.smooth_factors(O.calib_absmax(r_yA, 0), O.calib_absmax(WB, 1), 0.5)
    r_wqB, r_swB, _, _ = O.fold_quant_weights(WB, r_sB)
    r_swA2 = O.fold_next_smoothing(r_swA, r_sB)
    r_yA2 = O.w8a8_gemm(r_xqA, r_sxA, r_wqA, r_swA2, "bf16")
    r_xqB, r_sxB = O.ln_smooth_quant(r_yA2, s=np.ones(K2, np.float32))
    r_yB = O.w8a8_gemm(r_xqB, r_sxB, r_wqB, r_swB, "bf16")
    assert np.array_equal(host(sB), r_sB) and np.array_equal(host(swA2), r_swA2)
    assert np.array_equal(host(yA2), r_yA2)
    assert np.array_equal(host(rmax), O.calib_absmax(r_yA2, 1))
    assert np.array_equal(host(xqB), r_xqB) and np.array_equal(host(sxB), r_sxB)
    assert np.array_equal(host(yB), r_yB)

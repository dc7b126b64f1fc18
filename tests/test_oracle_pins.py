"""Pins for the CPU oracle: each test checks it against something other than itself --
values the pages print, closed forms, invariants, special cases that reduce to a
textbook routine, or brute force on tiny inputs.  CPU only.

Pages (title, section):
  [P3] "4.2 W8A8 量化与 SmoothQuant"
  [P4] "量化：只压权重，与训练后量化（PTQ）", SmoothQuant section and its worked example
  [P1] "大模型训练、适配与推理", sec. 3.5 SmoothQuant
  [P2] "SmoothQuant大模型平滑量化技术", Python demo
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import sq_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rel_fro(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


# ----------------------------------------------------------------------------- [P1] [P3 sec.3]
def test_equivalence_identity_fp64():
    """(X diag(s)^-1)(diag(s) W) = XW exactly in real arithmetic; fp64 to 1e-12 relative."""
    rng = np.random.default_rng(1)
    X = rng.standard_normal((37, 64))
    X[:, [3, 40]] *= 100.0
    W = rng.normal(0, 0.02, (64, 48))
    ax = O.calib_absmax(X.astype(np.float32), 0)
    aw = O.calib_absmax(W.astype(np.float32), 1)
    for alpha in (0.0, 0.4, 0.5, 0.75, 1.0):
        s = O.smooth_factors(ax, aw, alpha)
        Xs, Ws = O.smooth_transform_f64(X, W, s)
        assert _rel_fro(Xs @ Ws, X @ W) <= 1e-12


def test_smoothing_scales_the_input_channel_axis():
    """X' divides columns (input channels) and W' scales rows: a transposed fold breaks Y."""
    rng = np.random.default_rng(2)
    X = rng.standard_normal((5, 6))
    W = rng.standard_normal((6, 4))
    s = rng.uniform(0.5, 4.0, 6).astype(np.float32)
    Xs, Ws = O.smooth_transform_f64(X, W, s)
    assert np.allclose(Xs[:, 2] * s[2], X[:, 2])
    assert np.allclose(Ws[2, :] / s[2], W[2, :])


# ----------------------------------------------------------------------------- [P3 sec.4] [P4]
def test_alpha_half_balances_channel_maxima():
    """At alpha = 0.5 both smoothed channel maxima equal sqrt(max|X_j| * max|W_j|) [P4]."""
    c = sq_inputs.make_case(64, 128, 96, 3, x_dtype="f32", w_dtype="f32")
    ax = O.calib_absmax(c.x, 0)
    aw = O.calib_absmax(c.W, 1)
    s = O.smooth_factors(ax, aw, 0.5)
    Xs, Ws = O.smooth_transform_f64(c.x, c.W, s)
    target = np.sqrt(ax.astype(np.float64) * aw.astype(np.float64))
    assert np.allclose(np.abs(Xs).max(0), target, rtol=2e-7)
    assert np.allclose(np.abs(Ws).max(1), target, rtol=2e-7)


def test_alpha_extremes():
    """alpha = 1 -> s_j = max|X_j|: every smoothed activation channel max is exactly 1.
    alpha = 0 -> s_j = 1 / max|W_j|: every smoothed weight row max is 1 (within 1 ulp) [P3 sec.4]."""
    c = sq_inputs.make_case(32, 64, 48, 4, x_dtype="f32", w_dtype="f32")
    ax = O.calib_absmax(c.x, 0)
    aw = O.calib_absmax(c.W, 1)
    s1 = O.smooth_factors(ax, aw, 1.0)
    assert np.array_equal(s1, ax)
    assert np.array_equal(np.abs(c.x / s1[None, :]).max(0), np.ones(64, np.float32))
    s0 = O.smooth_factors(ax, aw, 0.0)
    wmax = np.abs(s0[:, None] * c.W).max(1)
    assert np.all(np.abs(wmax - 1.0) <= 2 * np.finfo(np.float32).eps)


def test_general_alpha_matches_power_form():
    """The exp/log path equals ax^a / aw^(1-a) evaluated with a different routine (pow)."""
    rng = np.random.default_rng(5)
    ax = rng.uniform(0.01, 500, 4096).astype(np.float32)
    aw = rng.uniform(1e-3, 0.2, 4096).astype(np.float32)
    for alpha in (0.4, 0.6, 0.75):
        s = O.smooth_factors(ax, aw, alpha)
        a = float(np.float32(alpha))
        ref = np.power(ax.astype(np.float64), a) / np.power(aw.astype(np.float64), 1.0 - a)
        ulp = np.spacing(ref.astype(np.float32))
        assert np.all(np.abs(s.astype(np.float64) - ref) <= ulp)
    # alpha = 0.5 shortcut agrees with the general form within 1 ulp
    s_half = O.smooth_factors(ax, aw, 0.5)
    ref = np.power(ax.astype(np.float64), 0.5) / np.power(aw.astype(np.float64), 0.5)
    assert np.all(np.abs(s_half - ref) <= np.spacing(s_half))


def test_alpha_half_scale_invariance():
    """s(c^2 ax) = c s(ax) at alpha = 0.5 for a power-of-two c (exact)."""
    rng = np.random.default_rng(6)
    ax = rng.uniform(0.1, 100, 512).astype(np.float32)
    aw = rng.uniform(0.01, 0.1, 512).astype(np.float32)
    s = O.smooth_factors(ax, aw, 0.5)
    s4 = O.smooth_factors(ax * 16.0, aw, 0.5)
    assert np.array_equal(s4, s * 4.0)


def test_zero_channel_convention():
    """Convention (unpinned by the pages): a channel with zero statistics keeps s = 1."""
    s = O.smooth_factors(np.array([0, 2, 3], np.float32), np.array([1, 0, 3], np.float32), 0.5)
    assert s.tolist() == [1.0, 1.0, 1.0]


# ----------------------------------------------------------------------------- [P3 sec.1.2]
def test_effective_levels_outlier_example():
    """One channel max 100, the rest in [-1, 1]: step 100/127 ~= 0.79, 2^8 * 1/100 = 2.56
    effective levels, and [-1, 1] lands on just the three codes {-1, 0, 1}."""
    rng = np.random.default_rng(7)
    y = rng.uniform(-1, 1, 1000).astype(np.float32)
    y[[0, 1]] = [1.0, -1.0]
    y[500] = 100.0
    q, scale = O.quant_per_tensor(y)
    assert scale == np.float32(100.0) / np.float32(127.0)
    assert abs(scale - 0.79) < 0.005
    small = np.delete(q, 500)
    assert set(np.unique(small).tolist()) == {-1, 0, 1}
    assert 2 ** 8 * 1.0 / 100.0 == pytest.approx(2.56)
    # the levels spanned by [-1, 1] out of the 255-code grid: 2^8 * m_i / m rounds to 3
    assert len(np.unique(small)) == round(2 ** 8 * 1.0 / 100.0)


# ----------------------------------------------------------------------------- [P4] worked example
def test_p4_worked_example():
    g = json.load(open(os.path.join(GOLDEN, "p4_worked_example.json")))
    X = np.array(g["X"], np.float32)
    W = np.array(g["W"], np.float32)
    ax = O.calib_absmax(X, 0)
    aw = O.calib_absmax(W, 1)
    assert np.allclose(ax, g["act_channel_absmax"]) and np.allclose(aw, g["weight_row_absmax"])
    s = O.smooth_factors(ax, aw, g["alpha"])
    assert np.all(np.abs(s - np.array(g["s"])) <= g["s_digits_abs"])
    Xs, Ws = O.smooth_transform_f64(X, W, s)
    for got in (np.abs(Xs).max(0), np.abs(Ws).max(1)):
        assert np.all(np.abs(got - np.array(g["smoothed_channel_max"])) <= g["smoothed_channel_max_abs"])

    Y = X.astype(np.float64) @ W.astype(np.float64)
    ones = np.ones(3, np.float32)
    errs_tensor, errs_token = [], []
    for i, sv in enumerate((ones, s)):
        wq, sw, _, _ = O.fold_quant_weights(W, sv)
        Xp = X / sv[None, :]
        q, scale = O.quant_per_tensor(Xp)
        step = g["per_tensor_step_before"] if i == 0 else g["per_tensor_step_after"]
        assert abs(scale - step) <= g["step_abs"]
        codes = g["channel0_codes_before"] if i == 0 else g["channel0_codes_after"]
        assert q[:, 0].tolist() == codes
        errs_tensor.append(_rel_fro(O.dequant_linear_f64(q, np.full(3, scale, np.float32), wq, sw), Y))
        xq, sx = O.ln_smooth_quant(X, s=sv)
        errs_token.append(_rel_fro(O.dequant_linear_f64(xq, sx, wq, sw), Y))
    assert np.all(np.abs(np.array(errs_tensor) - g["rel_err_per_tensor_act"]) <= g["rel_err_per_tensor_abs"])
    assert np.all(np.abs(np.array(errs_token) - g["rel_err_per_token_act"]) <= g["rel_err_per_token_abs"])


# ----------------------------------------------------------------------------- [P2] quantiser
def test_round_half_even_and_unit_scale():
    """absmax 127 gives scale exactly 1; ties go to even (2.5 -> 2, 3.5 -> 4, -2.5 -> -2)."""
    row = np.array([[2.5, 3.5, -2.5, 127.0, 0.5, 1.5, -0.5, -1.5]], np.float32)
    xq, sx = O.ln_smooth_quant(row, s=np.ones(8, np.float32))
    assert sx.tolist() == [1.0]
    assert xq.tolist() == [[2, 4, -2, 127, 0, 2, 0, -2]]


def test_per_token_codes_against_numpy_demo_rule():
    """The demo's rule (scale = max|x|/127, np.round = half-even, clip +-127) applied row by row."""
    rng = np.random.default_rng(8)
    x = rng.standard_normal((9, 64)).astype(np.float32)
    x[:, 5] *= 50
    xq, sx = O.ln_smooth_quant(x, s=np.ones(64, np.float32))
    for m in range(9):
        scale = np.float32(np.max(np.abs(x[m]))) / np.float32(127.0)
        ref = np.clip(np.round(x[m] / scale), -127, 127).astype(np.int8)
        assert sx[m] == scale
        assert np.array_equal(xq[m], ref)


def test_per_token_scale_is_per_row_and_scale_equivariant():
    """Per-token quantisation: scaling one row by 2^k leaves its codes and the others alone."""
    rng = np.random.default_rng(9)
    x = rng.standard_normal((6, 32)).astype(np.float32)
    ones = np.ones(32, np.float32)
    q0, s0 = O.ln_smooth_quant(x, s=ones)
    x2 = x.copy()
    x2[3] *= 8.0
    q1, s1 = O.ln_smooth_quant(x2, s=ones)
    assert np.array_equal(q0, q1)
    assert s1[3] == 8.0 * s0[3] and np.array_equal(np.delete(s1, 3), np.delete(s0, 3))


def test_zero_row_convention():
    xq, sx = O.ln_smooth_quant(np.zeros((2, 16), np.float32), s=np.ones(16, np.float32))
    assert sx.tolist() == [0.0, 0.0] and not xq.any()


# ----------------------------------------------------------------------------- weights [P3 sec.7.1]
def test_fold_quant_weights_per_output_channel():
    """Wq[k, :] dequantises to s_j W[j, k] within half a step, each nonzero column reaches 127,
    gamma' = gamma / s and beta' = beta / s."""
    c = sq_inputs.make_case(8, 96, 40, 10, x_dtype="f32", w_dtype="f32")
    rng = np.random.default_rng(11)
    s = rng.uniform(0.2, 8.0, 96).astype(np.float32)
    beta = rng.standard_normal(96).astype(np.float32)
    wq, sw, gf, bf = O.fold_quant_weights(c.W, s, c.gamma, beta)
    Wp = s[:, None].astype(np.float64) * c.W.astype(np.float64)          # [K, N]
    assert wq.shape == (40, 96)
    assert np.allclose(sw, np.abs(Wp).max(0) / 127.0, rtol=1e-6)
    deq = wq.astype(np.float64) * sw.astype(np.float64)[:, None]          # [N, K]
    assert np.all(np.abs(deq - Wp.T) <= sw[:, None] * 0.5 * (1 + 1e-5))
    assert np.all(np.abs(wq).max(1) == 127)
    assert np.allclose(gf, c.gamma / s, rtol=0, atol=0)
    assert np.allclose(bf, beta / s, rtol=0, atol=0)


def test_fold_bf16_input_matches_widened_fp32():
    c = sq_inputs.make_case(4, 64, 32, 12)
    s = np.random.default_rng(13).uniform(0.5, 3, 64).astype(np.float32)
    a = O.fold_quant_weights(c.W, s)
    b = O.fold_quant_weights(O.bf16_to_f32(c.W), s)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])


# ----------------------------------------------------------------------------- LayerNorm
def test_layernorm_reduces_to_textbook():
    """gamma = 1, beta = 0: the oracle's LN equals torch's fp64 layer_norm within 1e-6."""
    rng = np.random.default_rng(14)
    for K in (256, 4096, 14336):
        x = rng.standard_normal((3, K)).astype(np.float32)
        x[:, 7] *= 100
        y = O.layernorm(x, np.ones(K, np.float32), None, 1e-5)
        ref = torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (K,), eps=1e-5).numpy()
        assert np.max(np.abs(y - ref)) <= 1e-6 * max(1.0, np.max(np.abs(ref)))


def test_layernorm_affine_and_fold():
    """LN(x) diag(s)^-1 with folded gamma/s, beta/s equals LN(x)/s (within rounding) [P3 sec.6]."""
    rng = np.random.default_rng(15)
    K = 512
    x = rng.standard_normal((4, K)).astype(np.float32)
    gamma = rng.uniform(0.5, 1.5, K).astype(np.float32)
    beta = rng.normal(0, 0.1, K).astype(np.float32)
    s = rng.uniform(0.3, 20, K).astype(np.float32)
    ref = torch.nn.functional.layer_norm(torch.from_numpy(x).double(), (K,), torch.from_numpy(gamma).double(),
                                         torch.from_numpy(beta).double(), eps=1e-5).numpy()
    y = O.layernorm(x, gamma, beta)
    assert np.max(np.abs(y - ref)) <= 2e-6 * np.max(np.abs(ref))
    yf = O.layernorm(x, gamma / s, beta / s)
    assert np.max(np.abs(yf - ref / s)) <= 4e-6 * np.max(np.abs(ref / s))


def test_calib_ln_absmax_is_max_of_layernorm_output():
    c = sq_inputs.make_case(50, 256, 8, 16)
    ref = np.abs(O.layernorm(c.x, c.gamma)).max(0)
    got = O.calib_ln_absmax(c.x, c.gamma)
    assert np.array_equal(got, ref)
    half = O.calib_ln_absmax(c.x[:20], c.gamma)
    assert np.array_equal(O.calib_ln_absmax(c.x[20:], c.gamma, out=half), ref)


# ----------------------------------------------------------------------------- absmax
def test_calib_absmax_brute_force_and_accumulate():
    c = sq_inputs.make_case(33, 48, 40, 17)
    xf = O.bf16_to_f32(c.x)
    assert np.array_equal(O.calib_absmax(c.x, 0), np.abs(xf).max(0))
    wf = O.bf16_to_f32(c.W)
    assert np.array_equal(O.calib_absmax(c.W, 1), np.abs(wf).max(1))
    part = O.calib_absmax(c.x[:10], 0)
    assert np.array_equal(O.calib_absmax(c.x[10:], 0, out=part), np.abs(xf).max(0))


# ----------------------------------------------------------------------------- GEMM [P3 intro] [P4]
@pytest.mark.parametrize("M,N,K", [(1, 8, 16), (7, 24, 32), (32, 32, 256), (5, 3, 48)])
def test_int32_gemm_brute_force(M, N, K):
    rng = np.random.default_rng(M * 1000 + N + K)
    xq = rng.integers(-127, 128, (M, K), dtype=np.int64).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K), dtype=np.int64).astype(np.int8)
    xq[0, :] = 127
    wq[0, :] = -127
    acc = O.w8a8_gemm(xq, np.ones(M, np.float32), wq, np.ones(N, np.float32), "i32")
    ref = xq.astype(np.int64) @ wq.astype(np.int64).T
    assert np.array_equal(acc, ref)
    assert acc[0, 0] == -127 * 127 * K


def test_int32_accumulator_bound():
    """|acc| <= K * 127^2 fits int32 up to K = 133144, not beyond; the largest multiple of 16
    below it (133136) is the library's K limit."""
    assert 133144 * 127 * 127 <= 2 ** 31 - 1 < 133145 * 127 * 127
    assert 133136 % 16 == 0 and 133136 + 16 > 133144


def test_dequant_epilogue_against_torch():
    """bf16(((float)acc * sx) * sw), with torch doing the float32 arithmetic and the bf16 cast."""
    rng = np.random.default_rng(18)
    M, N, K = 9, 40, 64
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    wq = rng.integers(-127, 128, (N, K)).astype(np.int8)
    sx = rng.uniform(1e-3, 1, M).astype(np.float32)
    sw = rng.uniform(1e-4, 1e-2, N).astype(np.float32)
    y = O.w8a8_gemm(xq, sx, wq, sw, "bf16")
    acc = torch.from_numpy((xq.astype(np.int64) @ wq.astype(np.int64).T).astype(np.int32))
    ref = (acc.float() * torch.from_numpy(sx)[:, None]) * torch.from_numpy(sw)[None, :]
    assert np.array_equal(y, ref.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16))
    yf = O.w8a8_gemm(xq, sx, wq, sw, "f32")
    assert np.array_equal(yf, ref.numpy())


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(19)
    v = rng.standard_normal(2000).astype(np.float32) * np.float32(1e3)
    # exact ties and tie neighbours
    ties = (np.arange(64, dtype=np.uint32) << 16 | 0x8000).view(np.float32)
    v = np.concatenate([v, ties, np.array([0.0, -0.0, 1e38, 3.4e38], np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(O.f32_to_bf16(v), ref)


# ----------------------------------------------------------------------------- end to end
def test_pipeline_error_bound_tiny_case():
    """Dequantised W8A8 output of the whole path on the tiny outlier case stays within the
    per-element bound implied by half-step rounding of both operands, and smoothing
    reduces the error against the fp64 linear [P3 sec.3, P4]."""
    c = sq_inputs.tiny_case()
    ax = O.calib_absmax(c.x, 0)
    aw = O.calib_absmax(c.W, 1)
    Y = c.x.astype(np.float64) @ c.W.astype(np.float64)
    errs = {}
    for alpha in (None, 0.5):
        s = np.ones(c.K, np.float32) if alpha is None else O.smooth_factors(ax, aw, alpha)
        wq, sw, _, _ = O.fold_quant_weights(c.W, s)
        xq, sx = O.ln_smooth_quant(c.x, s=s)
        Yh = O.dequant_linear_f64(xq, sx, wq, sw)
        Xs, Ws = O.smooth_transform_f64(c.x, c.W, s)
        bound = (np.abs(Xs) @ np.ones((c.K, c.N))) * sw[None, :] * 0.5 \
            + sx[:, None] * 0.5 * (np.ones((c.M, c.K)) @ np.abs(Ws)) \
            + c.K * sx[:, None] * sw[None, :] * 0.25
        assert np.all(np.abs(Yh - Y) <= bound * (1 + 1e-4) + 1e-6)
        errs[alpha] = _rel_fro(Yh, Y)
    assert errs[0.5] < errs[None]


# ----------------------------------------------------------------------------- per-tensor granularity
def test_per_tensor_dynamic_matches_the_demo_rule_on_the_whole_tensor():
    """Per-tensor: the demo's quantize_int8 (one max/127 for the whole matrix) applied to y."""
    rng = np.random.default_rng(30)
    x = rng.standard_normal((7, 64)).astype(np.float32)
    x[:, 9] *= 80
    s = rng.uniform(0.5, 4.0, 64).astype(np.float32)
    xq, sx, scale = O.ln_smooth_quant_per_tensor(x, s=s)
    y = x / s[None, :]
    ref_scale = np.float32(np.max(np.abs(y))) / np.float32(127.0)
    assert scale == ref_scale and np.all(sx == ref_scale)
    assert np.array_equal(xq, np.clip(np.round(y / ref_scale), -127, 127).astype(np.int8))
    q2, s2 = O.quant_per_tensor(y)
    assert np.array_equal(q2, xq) and s2 == scale


def test_per_tensor_is_coarser_than_per_token():
    """The PTQ page's ladder: per-token activations quantise the outlier example more finely
    than one per-tensor scale (1.76% vs 1.95% without smoothing)."""
    g = json.load(open(os.path.join(GOLDEN, "p4_worked_example.json")))
    X = np.array(g["X"], np.float32)
    W = np.array(g["W"], np.float32)
    wq, sw, _, _ = O.fold_quant_weights(W, np.ones(3, np.float32))
    Y = X.astype(np.float64) @ W.astype(np.float64)
    qt, sxt, _ = O.ln_smooth_quant_per_tensor(X, s=np.ones(3, np.float32))
    qk, sxk = O.ln_smooth_quant(X, s=np.ones(3, np.float32))
    e_tensor = _rel_fro(O.dequant_linear_f64(qt, sxt, wq, sw), Y)
    e_token = _rel_fro(O.dequant_linear_f64(qk, sxk, wq, sw), Y)
    assert abs(e_tensor - g["rel_err_per_tensor_act"][0]) <= g["rel_err_per_tensor_abs"][0]
    assert e_token < e_tensor


def test_per_tensor_static_scale_clamps():
    """A calibrated scale smaller than this batch's max: codes saturate at +-127, the rest round."""
    x = np.array([[0.5, -300.0, 2.5, 1000.0, -1.5, 3.5, 0.0, 127.0]], np.float32)
    xq, sx, scale = O.ln_smooth_quant_per_tensor(x, s=np.ones(8, np.float32), static_scale=1.0)
    assert scale == 1.0 and sx.tolist() == [1.0]
    assert xq.tolist() == [[0, -127, 2, 127, -2, 4, 0, 127]]


def test_per_tensor_layernorm_mode_uses_the_same_layernorm():
    c = sq_inputs.make_case(6, 256, 8, 31, beta_std=0.1)
    y = O.layernorm(c.x, c.gamma, c.beta)
    xq, sx, scale = O.ln_smooth_quant_per_tensor(c.x, gamma_f=c.gamma, beta_f=c.beta)
    assert scale == np.float32(np.max(np.abs(y))) / np.float32(127.0)
    q2, _ = O.quant_per_tensor(y)
    assert np.array_equal(xq, q2)


# ----------------------------------------------------------------------------- FP8 (E4M3) variant
# The pages name FP8 W8A8 (the FP8 tensor-core peak is twice BF16's) without fixing the
# encoding; the reading is E4M3 of the OCP 8-bit floating point specification, and these
# pins hold the oracle's encoder and decoder to torch's float8_e4m3fn, an independent
# implementation of the same format.
def _torch_e4m3(v: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(v, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_decode_every_code_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    got = O.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    fin = ~np.isnan(ref)
    assert np.array_equal(got[fin].view(np.uint32), ref[fin].view(np.uint32))
    assert np.isnan(got).sum() == 2 and got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9


def test_e4m3_encode_grid_midpoints_and_random_values_match_torch():
    grid = O.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8)).astype(np.float64)  # 0 .. 448
    mids = (grid[:-1] + grid[1:]) / 2                      # ties: nearest even code
    quarter = grid[:-1] + (grid[1:] - grid[:-1]) / 4
    rng = np.random.default_rng(3)
    rand = np.concatenate([rng.uniform(0, 463.9, 4000), np.exp(rng.uniform(np.log(2.0 ** -12), np.log(463.0), 4000))])
    v = np.concatenate([grid, mids, quarter, rand]).astype(np.float32)
    v = np.concatenate([v, -v])
    assert np.array_equal(O.e4m3_encode(v), _torch_e4m3(v))
    assert np.array_equal(O.e4m3_encode(O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))), np.arange(0x7F))


def test_e4m3_saturates_at_the_largest_finite_value():
    v = np.array([448.0, 463.9, 464.0, 500.0, 1e30, -470.0], np.float32)
    assert O.e4m3_encode(v).tolist() == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE]


def test_fp8_fold_per_output_channel():
    c = sq_inputs.make_case(4, 96, 40, 12)
    s = np.exp(np.random.default_rng(4).uniform(-1, 1, 96)).astype(np.float32)
    wq, sw, _, _ = O.fold_quant_weights_fp8(c.W, s)
    Wp = (s[:, None] * O.bf16_to_f32(c.W)).astype(np.float32)          # W' = diag(s) W, [K, N]
    assert np.array_equal(sw, np.max(np.abs(Wp), axis=0) / np.float32(448.0))
    dec = O.e4m3_decode(wq).astype(np.float64)                           # [N, K]
    assert np.all(np.max(np.abs(dec), axis=1) == 448.0)                  # every column reaches the top code
    err = np.abs(dec * sw[:, None] - Wp.T.astype(np.float64))
    # half an E4M3 step: 2^-4 relative for normal codes, 2^-10 of the scale below 2^-6
    assert np.all(err <= np.maximum(np.abs(Wp.T) * 2.0 ** -4, 2.0 ** -10 * sw[:, None]) * (1 + 1e-6))


def test_fp8_per_token_codes_follow_the_definition():
    c = sq_inputs.make_case(9, 128, 8, 13)
    s = np.exp(np.random.default_rng(5).uniform(-1, 2, 128)).astype(np.float32)
    xq, sx = O.ln_smooth_quant_fp8(c.x, s=s)
    y = (O.bf16_to_f32(c.x) / s[None, :]).astype(np.float32)
    ref_sx = np.max(np.abs(y), axis=1) / np.float32(448.0)
    assert np.array_equal(sx, ref_sx)
    q = (y / ref_sx[:, None]).astype(np.float32)
    assert np.array_equal(xq, _torch_e4m3(q))                            # |q| <= 448: torch's rounding applies
    xl, sl = O.ln_smooth_quant_fp8(c.x, gamma_f=c.gamma)
    yl = O.layernorm(c.x, c.gamma)
    assert np.array_equal(sl, np.max(np.abs(yl), axis=1) / np.float32(448.0))
    assert np.array_equal(xl, _torch_e4m3((yl / sl[:, None]).astype(np.float32)))


@pytest.mark.parametrize("M,N,K", [(1, 1, 16), (3, 5, 64), (7, 6, 200)])
def test_fp8_gemm_accumulator_is_the_exact_sum(M, N, K):
    import fractions
    rng = np.random.default_rng(M * N + K)
    fin = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    xq = rng.choice(fin, (M, K)).astype(np.uint8)
    wq = rng.choice(fin, (N, K)).astype(np.uint8)
    xq[0, :4] = 0x7E
    wq[0, :4] = 0xFE                                                     # -448 * 448 products
    acc, y = O.fp8_gemm(xq, np.ones(M, np.float32), wq, np.ones(N, np.float32), "f32")
    dx, dw = O.e4m3_decode(xq), O.e4m3_decode(wq)
    for m in range(M):
        for n in range(N):
            exact = sum(fractions.Fraction(float(a)) * fractions.Fraction(float(b)) for a, b in zip(dx[m], dw[n]))
            assert fractions.Fraction(acc[m, n]) == exact
            assert y[m, n] == np.float32(float(exact))


def test_fp8_smoothquant_linear_error_is_small():
    """Smoothing + E4M3 codes on the outlier case: the dequantised linear stays within a few
    E4M3 steps of XW (3 mantissa bits: per-element error below 2^-4 relative)."""
    c = sq_inputs.tiny_case()
    x = O.bf16_to_f32(c.x) if c.x.dtype == np.uint16 else c.x
    W = O.bf16_to_f32(c.W) if c.W.dtype == np.uint16 else c.W
    s = O.smooth_factors(O.calib_absmax(x, 0), O.calib_absmax(W, 1), 0.5)
    wq, sw, _, _ = O.fold_quant_weights_fp8(W, s)
    xq, sx = O.ln_smooth_quant_fp8(x, s=s)
    acc, _ = O.fp8_gemm(xq, sx, wq, sw, "f32")
    yq = acc * sx[:, None].astype(np.float64) * sw[None, :].astype(np.float64)
    Y = x.astype(np.float64) @ W.astype(np.float64)
    assert _rel_fro(yq, Y) < 2.0 ** -4


# ----------------------------------------------------------------------------- alpha search
def test_alpha_search_objective_reproduces_the_worked_example():
    """The objective at alpha = 0.5 on the PTQ page's 3x3 example is the square of the page's
    per-token relative error after smoothing (0.048%)."""
    g = json.load(open(os.path.join(GOLDEN, "p4_worked_example.json")))
    X = np.array(g["X"], np.float32)
    W = np.array(g["W"], np.float32)
    err = O.alpha_search(X, W, [0.5])
    rel = float(np.sqrt(err[0]))
    want, tol = g["rel_err_per_token_act"][1], g["rel_err_per_token_abs"][1]
    assert abs(rel - want) <= tol, (rel, want)


def test_alpha_search_grid_and_extremes():
    """20 strengths over [0, 1]; on an outlier-bearing case neither extreme is the optimum
    (alpha = 0 leaves the activation outliers, alpha = 1 moves them all into the weights)."""
    a = O.alpha_grid(20)
    assert a.size == 20 and a[0] == 0.0 and a[-1] == 1.0 and np.all(np.diff(a) > 0)
    c = sq_inputs.make_case(96, 256, 64, 21, outlier_mult=60.0)
    err = O.alpha_search(c.x, c.W, a, gamma=c.gamma)
    best = int(np.argmin(err))
    assert 0 < best < a.size - 1
    assert err[best] < 0.5 * min(err[0], err[-1])


# ----------------------------------------------------------------------------- smoothing folded into the previous linear
def _two_layer_chain(seed, folded):
    """Linear A (K1 -> K2, plain input) feeding linear B (K2 -> N); B's smoothing either divides
    its input at run time (plain mode, s_B) or is folded into A's output scales."""
    rng = np.random.default_rng(seed)
    M, K1, K2, N = 40, 128, 96, 64
    x = (rng.standard_normal((M, K1)) * np.where(rng.random(K1) < 0.03, 30.0, 1.0)).astype(np.float32)
    WA = rng.normal(0, 0.05, (K1, K2)).astype(np.float32)
    WB = rng.normal(0, 0.05, (K2, N)).astype(np.float32)
    sA = O.smooth_factors(O.calib_absmax(x, 0), O.calib_absmax(WA, 1), 0.5)
    wqA, swA, _, _ = O.fold_quant_weights(WA, sA)
    xqA, sxA = O.ln_smooth_quant(x, s=sA)
    yA = O.w8a8_gemm(xqA, sxA, wqA, swA, "f32")                     # B's input, unsmoothed
    sB = O.smooth_factors(O.calib_absmax(yA, 0), O.calib_absmax(WB, 1), 0.5)
    wqB, swB, _, _ = O.fold_quant_weights(WB, sB)
    if folded:
        yA = O.w8a8_gemm(xqA, sxA, wqA, O.fold_next_smoothing(swA, sB), "f32")   # already y / sB
        xqB, sxB = O.ln_smooth_quant(yA, s=np.ones(K2, np.float32))
    else:
        xqB, sxB = O.ln_smooth_quant(yA, s=sB)
    return O.w8a8_gemm(xqB, sxB, wqB, swB, "f32"), xqB


def test_fold_next_smoothing_divides_the_output_channel_scale():
    rng = np.random.default_rng(8)
    sw = np.exp(rng.uniform(-10, 0, 64)).astype(np.float32)
    s = np.exp(rng.uniform(-2, 3, 64)).astype(np.float32)
    out = O.fold_next_smoothing(sw, s)
    assert np.array_equal(out, (sw / s).astype(np.float32))
    # the dequantised output with the folded scale is y / s within two binary32 roundings
    acc = rng.integers(-2 ** 20, 2 ** 20, (8, 64)).astype(np.float64)
    sx = np.exp(rng.uniform(-6, 0, 8)).astype(np.float32)
    y = ((acc.astype(np.float32) * sx[:, None]).astype(np.float32) * sw[None, :]).astype(np.float32)
    y2 = ((acc.astype(np.float32) * sx[:, None]).astype(np.float32) * out[None, :]).astype(np.float32)
    ref = y.astype(np.float64) / s[None, :].astype(np.float64)
    assert np.all(np.abs(y2 - ref) <= 4 * np.spacing(np.abs(ref).astype(np.float32)))


def test_folded_chain_matches_the_runtime_division():
    """Folding B's smoothing into A changes only roundings: B's codes agree almost everywhere and
    B's output stays within a fraction of its quantisation error."""
    y_rt, q_rt = _two_layer_chain(3, folded=False)
    y_fd, q_fd = _two_layer_chain(3, folded=True)
    assert (q_rt == q_fd).mean() > 0.99
    assert np.linalg.norm(y_fd - y_rt) / np.linalg.norm(y_rt) < 2e-3

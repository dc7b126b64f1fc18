"""GPU parity: every call of the CUDA library (through the C ABI) against the CPU oracle on
the same seeded bytes.  Bar: bit-exact for absmax statistics, smoothing factors, scales,
int8 codes and int32 accumulators; bf16 outputs within 1 bf16 ulp or 4e-3 relative (the
kernels take the oracle's exact sequence of roundings, so they are in fact bit-identical,
which the tests also record).  Small cases are compared in full; full-size workloads on
sampled rows (every column of those rows)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
import sq_inputs
import w8a8_smoothquant_gemm_b200 as sq

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


# ----------------------------------------------------------------------------- helpers
def dev(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


def host(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def assert_bf16_close(got_bits: np.ndarray, ref_bits: np.ndarray):
    """Within 1 bf16 ulp or 4e-3 relative; returns the bit-identical fraction."""
    g = O.bf16_to_f32(got_bits).astype(np.float64)
    r = O.bf16_to_f32(ref_bits).astype(np.float64)
    ulp = np.spacing(np.abs(r).astype(np.float32)).astype(np.float64) * 65536.0  # bf16 ulp = 2^16 f32 ulps
    ok = (np.abs(g - r) <= ulp) | (np.abs(g - r) <= 4e-3 * np.abs(r))
    assert ok.all(), f"{(~ok).sum()} bf16 outputs outside tolerance"
    return float((got_bits == ref_bits).mean())


def padded(a: np.ndarray, extra: int) -> np.ndarray:
    """Same values in a wider buffer (leading dimension = cols + extra)."""
    out = np.zeros((a.shape[0], a.shape[1] + extra), a.dtype)
    out[:, : a.shape[1]] = a
    return out


@pytest.fixture(autouse=True)
def _no_device_error():
    sq.sq_device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert sq.sq_device_error(clear=True) == 0


# ----------------------------------------------------------------------------- tiny config, whole path
def test_tiny_config_full_path():
    """16 x 256 -> 256, fp32, 3 outlier channels x100, alpha 0.5, calibration on X itself."""
    c = sq_inputs.tiny_case()
    x, W = dev(c.x), dev(c.W)
    ax = sq.sq_calib_absmax(x, 0)
    aw = sq.sq_calib_absmax(W, 1)
    s = sq.sq_smooth_factors(ax, aw, 0.5)
    wq, sw, _, _ = sq.sq_fold_quant_weights(W, s)
    xq, sx = sq.sq_ln_smooth_quant(x, s=s)
    y = sq.sq_w8a8_gemm(xq, sx, wq, sw)
    acc = sq.sq_w8a8_gemm(xq, None, wq, None, out_dtype=torch.int32)

    r_ax, r_aw = O.calib_absmax(c.x, 0), O.calib_absmax(c.W, 1)
    r_s = O.smooth_factors(r_ax, r_aw, 0.5)
    r_wq, r_sw, _, _ = O.fold_quant_weights(c.W, r_s)
    r_xq, r_sx = O.ln_smooth_quant(c.x, s=r_s)
    assert np.array_equal(host(ax), r_ax) and np.array_equal(host(aw), r_aw)
    assert np.array_equal(host(s), r_s)
    assert np.array_equal(host(wq), r_wq) and np.array_equal(host(sw), r_sw)
    assert np.array_equal(host(xq), r_xq) and np.array_equal(host(sx), r_sx)
    assert np.array_equal(host(acc), O.w8a8_gemm(r_xq, r_sx, r_wq, r_sw, "i32"))
    assert assert_bf16_close(host(y), O.w8a8_gemm(r_xq, r_sx, r_wq, r_sw, "bf16")) == 1.0


# ----------------------------------------------------------------------------- calibration absmax
@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("rows,cols,extra", [(1, 8, 0), (3, 64, 8), (1000, 4096, 0), (257, 136, 24), (4097, 520, 0)])
def test_calib_absmax(dt, rows, cols, extra):
    c = sq_inputs.make_case(rows, cols, 8, rows + cols, x_dtype=dt, w_dtype=dt)
    cols_f32_ok = dt == "bf16" or cols % 4 == 0
    assert cols_f32_ok
    xh = padded(c.x, extra)
    xd = dev(xh)[:, :cols]
    got0 = sq.sq_calib_absmax(xd, 0)
    got1 = sq.sq_calib_absmax(xd, 1)
    assert np.array_equal(host(got0), O.calib_absmax(c.x, 0))
    assert np.array_equal(host(got1), O.calib_absmax(c.x, 1))
    # accumulate over two batches equals one pass
    half = rows // 2
    part = sq.sq_calib_absmax(xd[:half], 0) if half else torch.zeros(cols, device=DEV)
    sq.sq_calib_absmax(xd[half:], 0, out=part, accumulate=True)
    assert np.array_equal(host(part), O.calib_absmax(c.x, 0))
    prev = torch.full((rows,), 3.0, device=DEV)
    sq.sq_calib_absmax(xd, 1, out=prev, accumulate=True)
    assert np.array_equal(host(prev), np.maximum(O.calib_absmax(c.x, 1), 3.0).astype(np.float32))


def test_calibration_config_full_size():
    """512 x 512 tokens x K = 4096 bf16 with ~1% channels x log-uniform[20, 100]; W [4096, 4096];
    s for alpha in {0.4, 0.5, 0.6, 0.75}."""
    x, W, _, _ = sq_inputs.torch_case(512 * 512, 4096, 4096, 1, DEV, outlier_mult=(20.0, 100.0))
    ax = sq.sq_calib_absmax(x, 0)
    aw = sq.sq_calib_absmax(W, 1)
    xh, wh = host(x), host(W)
    del x
    torch.cuda.empty_cache()
    r_ax, r_aw = O.calib_absmax(xh, 0), O.calib_absmax(wh, 1)
    assert np.array_equal(host(ax), r_ax) and np.array_equal(host(aw), r_aw)
    for alpha in (0.4, 0.5, 0.6, 0.75):
        assert np.array_equal(host(sq.sq_smooth_factors(ax, aw, alpha)), O.smooth_factors(r_ax, r_aw, alpha))


# ----------------------------------------------------------------------------- smoothing factors
@pytest.mark.parametrize("alpha", [0.0, 0.25, 0.4, 0.5, 0.6, 0.75, 0.9, 1.0])
def test_smooth_factors(alpha):
    rng = np.random.default_rng(3)
    K = 65536
    ax = np.exp(rng.uniform(-8, 8, K)).astype(np.float32)
    aw = np.exp(rng.uniform(-10, 2, K)).astype(np.float32)
    ax[:5] = 0.0
    aw[5:9] = 0.0
    got = sq.sq_smooth_factors(dev(ax), dev(aw), alpha)
    assert np.array_equal(host(got), O.smooth_factors(ax, aw, alpha))


# ----------------------------------------------------------------------------- fold + weight quant
@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("K,N,extra", [(16, 8, 0), (256, 256, 0), (272, 200, 8), (4096, 4096, 0), (1040, 3000, 0)])
def test_fold_quant_weights(dt, K, N, extra):
    c = sq_inputs.make_case(4, K, N, K + N, x_dtype=dt, w_dtype=dt, beta_std=0.1)
    if N > 3:
        c.W[:, 3] = 0  # an all-zero output channel: scale 0, codes 0
    rng = np.random.default_rng(K)
    s = np.exp(rng.uniform(-2, 3, K)).astype(np.float32)
    Wh = padded(c.W, extra)
    Wd = dev(Wh)[:, :N]
    wq, sw, gf, bf = sq.sq_fold_quant_weights(Wd, dev(s), dev(c.gamma), dev(c.beta))
    r = O.fold_quant_weights(c.W, s, c.gamma, c.beta)
    assert np.array_equal(host(wq), r[0])
    assert np.array_equal(host(sw), r[1])
    assert np.array_equal(host(gf), r[2]) and np.array_equal(host(bf), r[3])


@pytest.mark.parametrize("K,N,extra", [(40000, 1288, 8), (49168, 1096, 0), (16, 3145800, 0)])
def test_fold_streaming_ragged(K, N, extra):
    """The streaming two-pass route on a ragged last row tile and column strip, with a padded
    leading dimension and an all-zero output channel; K = 16 is a single, mostly empty row
    tile under a 100 MB wide weight."""
    _, W, g, _ = sq_inputs.torch_case(1, K, N, 11, DEV, w_std=0.015)
    W = torch.nn.functional.pad(W, (0, extra))[:, :N] if extra else W
    W[:, 5] = 0
    assert sq.sq_fold_kernel_launches(W) == 3
    rng = np.random.default_rng(K + N)
    s = np.exp(rng.uniform(-1, 2, K)).astype(np.float32)
    wq, sw, gf, _ = sq.sq_fold_quant_weights(W, dev(s), g)
    r_wq, r_sw, r_gf, _ = O.fold_quant_weights(host(W), s, host(g))
    assert np.array_equal(host(sw), r_sw)
    assert np.array_equal(host(wq), r_wq)
    assert np.array_equal(host(gf), r_gf)


@pytest.mark.parametrize("K,N", [(4096, 28672), (14336, 4096), (49152, 12288)])
def test_fold_full_size(K, N):
    _, W, _, _ = sq_inputs.torch_case(1, K, N, 7, DEV, w_std=0.015)
    rng = np.random.default_rng(K)
    s = np.exp(rng.uniform(-1, 2, K)).astype(np.float32)
    wq, sw, _, _ = sq.sq_fold_quant_weights(W, dev(s))
    r_wq, r_sw, _, _ = O.fold_quant_weights(host(W), s)
    assert np.array_equal(host(sw), r_sw)
    assert np.array_equal(host(wq), r_wq)


# ----------------------------------------------------------------------------- LN + smooth + quant
@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("M,K", [(1, 16), (5, 256), (9, 1040), (33, 2048), (64, 4096), (7, 8192), (3, 12288),
                                 (17, 14336), (4, 16384), (3, 16400), (2, 49152), (37, 20000), (513, 24576)])
@pytest.mark.parametrize("mode", ["ln", "plain"])
def test_ln_smooth_quant(dt, M, K, mode):
    if dt == "f32" and K > 32768:
        pytest.skip("fp32 rows are limited to K <= 32768")
    c = sq_inputs.make_case(M, K, 8, M * 7 + K, x_dtype=dt, w_dtype=dt, beta_std=0.05)
    rng = np.random.default_rng(K + 1)
    s = np.exp(rng.uniform(-1, 3, K)).astype(np.float32)
    xh = padded(c.x, 16)
    xd = dev(xh)[:, :K]
    if M > 1:
        c.x[1] = 0  # an all-zero row: scale 0 and zero codes (plain mode); LN of a zero row is beta
        xd[1] = 0
    if mode == "ln":
        gf, bf = (c.gamma / s).astype(np.float32), (c.beta / s).astype(np.float32)
        xq, sx = sq.sq_ln_smooth_quant(xd, gamma_f=dev(gf), beta_f=dev(bf))
        r_xq, r_sx = O.ln_smooth_quant(c.x, gamma_f=gf, beta_f=bf)
    else:
        xq, sx = sq.sq_ln_smooth_quant(xd, s=dev(s))
        r_xq, r_sx = O.ln_smooth_quant(c.x, s=s)
    assert np.array_equal(host(sx), r_sx)
    assert np.array_equal(host(xq), r_xq)


@pytest.mark.parametrize("rows,K", [(1, 256), (100, 4096), (1000, 4096), (70, 8192), (5, 14336), (33, 49152),
                                    (20, 12288), (9, 10240), (300, 24576)])
def test_calib_ln_absmax(rows, K):
    c = sq_inputs.make_case(rows, K, 8, rows + K, beta_std=0.1)
    got = sq.sq_calib_ln_absmax(dev(c.x), dev(c.gamma), dev(c.beta))
    assert np.array_equal(host(got), O.calib_ln_absmax(c.x, c.gamma, c.beta))
    sq.sq_calib_ln_absmax(dev(c.x), dev(c.gamma), dev(c.beta), out=got, accumulate=True)
    assert np.array_equal(host(got), O.calib_ln_absmax(c.x, c.gamma, c.beta))


# ----------------------------------------------------------------------------- prefill-sized row counts
# From about a thousand rows on, rows of the model widths go to one-warp-per-row kernels
# (chunk pairs on packed binary32); these cases cover every width they take, with a ragged
# row count, a padded leading dimension and the degenerate rows.
PAIR_WIDTHS = [512, 1024, 2048, 4096, 8192, 12288, 14336]


def _many_rows(M, K, seed):
    c = sq_inputs.make_case(M, K, 8, seed, beta_std=0.05)
    c.x[1] = 0  # all-zero row
    # a row of tiny values: in plain mode its scale falls below 2^-90, where the shared-divisor
    # quotient takes the correctly rounded division instead
    c.x[2] = sq_inputs.to_bf16_bits(O.bf16_to_f32(c.x[2]) * np.float32(2.0 ** -100))
    return c


@pytest.mark.parametrize("K", PAIR_WIDTHS)
@pytest.mark.parametrize("mode", ["ln", "plain"])
def test_ln_smooth_quant_many_rows(K, mode):
    M = 1031
    c = _many_rows(M, K, 11 * K + 3)
    s = np.exp(np.random.default_rng(K + 5).uniform(-1, 3, K)).astype(np.float32)
    xd = dev(padded(c.x, 16))[:, :K]
    if mode == "ln":
        gf, bf = (c.gamma / s).astype(np.float32), (c.beta / s).astype(np.float32)
        xq, sx = sq.sq_ln_smooth_quant(xd, gamma_f=dev(gf), beta_f=dev(bf))
        r_xq, r_sx = O.ln_smooth_quant(c.x, gamma_f=gf, beta_f=bf)
    else:
        xq, sx = sq.sq_ln_smooth_quant(xd, s=dev(s))
        r_xq, r_sx = O.ln_smooth_quant(c.x, s=s)
        assert r_sx[2] < 2.0 ** -90 and r_sx[1] == 0
    assert np.array_equal(host(sx), r_sx)
    assert np.array_equal(host(xq), r_xq)


@pytest.mark.parametrize("K", [4096, 14336])
def test_plain_quant_many_rows_divisor_outside_fast_range(K):
    """A smoothing factor below 2^-90: every division of that launch is correctly rounded."""
    M = 1030
    c = _many_rows(M, K, K + 17)
    s = np.exp(np.random.default_rng(K + 6).uniform(-1, 3, K)).astype(np.float32)
    s[5] = np.float32(2.0 ** -100)
    xq, sx = sq.sq_ln_smooth_quant(dev(c.x), s=dev(s))
    r_xq, r_sx = O.ln_smooth_quant(c.x, s=s)
    assert np.array_equal(host(sx), r_sx)
    assert np.array_equal(host(xq), r_xq)


@pytest.mark.parametrize("K", PAIR_WIDTHS)
@pytest.mark.parametrize("mode", ["ln", "plain"])
def test_per_tensor_many_rows(K, mode):
    """Per-tensor scales (dynamic, then static at half of it: clamping) through the same kernels."""
    M = 1029
    c = sq_inputs.make_case(M, K, 8, 13 * K + 1, beta_std=0.05)
    s = np.exp(np.random.default_rng(K + 7).uniform(-1, 3, K)).astype(np.float32)
    kw = dict(gamma_f=(c.gamma / s).astype(np.float32)) if mode == "ln" else dict(s=s)
    dkw = {k: dev(v) for k, v in kw.items()}
    xq, sx, sc = sq.sq_ln_smooth_quant_per_tensor(dev(c.x), **dkw)
    r_xq, r_sx, r_sc = O.ln_smooth_quant_per_tensor(c.x, **kw)
    assert host(sc)[0] == np.float32(r_sc)
    assert np.array_equal(host(sx), r_sx) and np.array_equal(host(xq), r_xq)
    static = np.float32(r_sc * 0.5)
    xq, sx, _ = sq.sq_ln_smooth_quant_per_tensor(dev(c.x), scale=dev(np.array([static], np.float32)), static=True,
                                                 **dkw)
    r_xq, r_sx, _ = O.ln_smooth_quant_per_tensor(c.x, static_scale=float(static), **kw)
    assert np.array_equal(host(sx), r_sx) and np.array_equal(host(xq), r_xq)
    assert (np.abs(r_xq) == 127).sum() > 0


@pytest.mark.parametrize("rows,K", [(1030, 512), (1100, 1024), (1027, 2048), (2051, 4096), (1500, 8192),
                                    (2048, 12288), (2051, 14336)])
def test_calib_ln_absmax_many_rows(rows, K):
    c = _many_rows(rows, K, rows + 3 * K)
    x = dev(padded(c.x, 8))[:, :K]
    got = sq.sq_calib_ln_absmax(x, dev(c.gamma), dev(c.beta))
    ref = O.calib_ln_absmax(c.x, c.gamma, c.beta)
    assert np.array_equal(host(got), ref)
    sq.sq_calib_ln_absmax(x, dev(c.gamma), dev(c.beta), out=got, accumulate=True)
    assert np.array_equal(host(got), ref)


# ----------------------------------------------------------------------------- GEMM
def random_codes(rng, rows, K, extreme_row=None):
    q = rng.integers(-127, 128, (rows, K), dtype=np.int64).astype(np.int8)
    if extreme_row is not None and rows > 0:
        q[extreme_row] = extreme_row % 2 and -127 or 127
    return q


GEMM_SHAPES = [
    (1, 8, 16), (1, 200, 272), (7, 24, 32), (16, 256, 256), (33, 4096, 4096), (64, 130, 1024),
    (100, 1000, 512), (128, 512, 128), (129, 264, 128), (200, 777, 400), (256, 512, 4096),
    (300, 1024, 1040), (1000, 300, 160), (2048, 512, 96),
    (5, 1000, 8192), (7, 5120, 2048),  # decode shapes split 16 and 3 ways
    # decode shapes whose weight tiles are shared by several CTAs (stream-K): 1.5 tiles per CTA,
    # 128-token columns, ~5 CTAs per tile over a long K, and two full waves of whole tiles
    (1, 28672, 4096), (128, 12288, 1024), (16, 4096, 49152), (2, 36864, 256),
    # whole tiles in a full wave plus one tile split over a few CTAs (most CTAs' split ranges empty),
    # and two full waves plus a split remainder
    (1, 19072, 272), (64, 40960, 1024),
    # CTA-pair tiles over several waves, one with a ragged last column tile
    (2048, 12288, 256), (2048, 12200, 128),
]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_gemm_int32_and_epilogue(M, N, K):
    rng = np.random.default_rng(M * 31 + N * 7 + K)
    xq = random_codes(rng, M, K, extreme_row=0)
    wq = random_codes(rng, N, K, extreme_row=min(1, N - 1))
    sx = rng.uniform(1e-3, 0.5, M).astype(np.float32)
    sw = rng.uniform(1e-5, 1e-2, N).astype(np.float32)
    dx, dw, dsx, dsw = dev(xq), dev(wq), dev(sx), dev(sw)
    acc = sq.sq_w8a8_gemm(dx, None, dw, None, out_dtype=torch.int32)
    assert np.array_equal(host(acc), O.w8a8_gemm(xq, sx, wq, sw, "i32"))
    yb = sq.sq_w8a8_gemm(dx, dsx, dw, dsw)
    assert assert_bf16_close(host(yb), O.w8a8_gemm(xq, sx, wq, sw, "bf16")) == 1.0
    yf = sq.sq_w8a8_gemm(dx, dsx, dw, dsw, out_dtype=torch.float32)
    assert np.array_equal(host(yf), O.w8a8_gemm(xq, sx, wq, sw, "f32"))


def test_gemm_output_leading_dimension():
    rng = np.random.default_rng(11)
    M, N, K = 150, 96, 256
    xq, wq = random_codes(rng, M, K), random_codes(rng, N, K)
    sx = rng.uniform(1e-3, 1, M).astype(np.float32)
    sw = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    ybuf = torch.full((M, N + 40), -1.0, dtype=torch.bfloat16, device=DEV)
    sq.sq_w8a8_gemm(dev(xq), dev(sx), dev(wq), dev(sw), y=ybuf[:, :N])
    assert assert_bf16_close(host(ybuf[:, :N].contiguous()), O.w8a8_gemm(xq, sx, wq, sw, "bf16")) == 1.0
    assert (host(ybuf[:, N:].float()) == -1.0).all()


def test_gemm_workspace_reused_across_calls_and_shapes():
    """One zero-filled workspace serves calls of different shapes in turn (stream-K tile sums,
    split-K partials): all of it is back at zero after every call, and every result is exact."""
    shapes = [(16, 4096, 4096), (1, 28672, 4096), (64, 6144, 4096), (16, 4096, 4096), (3, 1000, 14336),
              (256, 512, 4096), (1, 28672, 4096)]
    need = max(sq.sq_w8a8_gemm_workspace_size(*sh) for sh in shapes)
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    rng = np.random.default_rng(5)
    for M, N, K in shapes:
        xq, wq = random_codes(rng, M, K, extreme_row=0), random_codes(rng, N, K)
        acc = sq.sq_w8a8_gemm(dev(xq), None, dev(wq), None, out_dtype=torch.int32, workspace=ws)
        assert np.array_equal(host(acc), O.w8a8_gemm(xq, None, wq, None, "i32"))
        assert not ws.any()


def test_gemm_workspace_too_small_is_reported():
    M, N, K = 1, 4096, 4096
    need = sq.sq_w8a8_gemm_workspace_size(M, N, K)
    assert need > 0  # decode shapes split K across SMs
    xq = torch.zeros(M, K, dtype=torch.int8, device=DEV)
    wq = torch.zeros(N, K, dtype=torch.int8, device=DEV)
    small = torch.empty(need // 2, dtype=torch.uint8, device=DEV)
    with pytest.raises(sq.SQError) as ei:
        sq.sq_w8a8_gemm(xq, None, wq, None, out_dtype=torch.int32, workspace=small)
    assert ei.value.status == 5


def _layer(M, K, N, seed, w_std, ln):
    """A full linear: calibration on the batch, alpha = 0.5, fold, quantise, GEMM -- on the GPU
    and in the oracle; returns both sides' intermediates."""
    x, W, gamma, _ = sq_inputs.torch_case(M, K, N, seed, DEV, w_std=w_std)
    if ln:
        ax = sq.sq_calib_ln_absmax(x, gamma)
    else:
        ax = sq.sq_calib_absmax(x, 0)
    aw = sq.sq_calib_absmax(W, 1)
    s = sq.sq_smooth_factors(ax, aw, 0.5)
    wq, sw, gf, _ = sq.sq_fold_quant_weights(W, s, gamma if ln else None)
    xq, sx = sq.sq_ln_smooth_quant(x, gamma_f=gf) if ln else sq.sq_ln_smooth_quant(x, s=s)
    y = sq.sq_w8a8_gemm(xq, sx, wq, sw)
    return dict(x=host(x), W=host(W), gamma=host(gamma), ax=host(ax), aw=host(aw), s=host(s), wq=host(wq),
                sw=host(sw), gf=host(gf) if ln else None, xq=host(xq), sx=host(sx), y=host(y))


DECODE = [(M, K, N, ln) for M in (1, 16, 64)
          for (K, N, ln) in ((4096, 6144, True), (4096, 4096, False), (4096, 28672, True), (14336, 4096, False))]


@pytest.mark.parametrize("M,K,N,ln", DECODE)
def test_decode_layer_full(M, K, N, ln):
    g = _layer(M, K, N, 100 + M + N, 0.02, ln)
    ax = O.calib_ln_absmax(g["x"], g["gamma"]) if ln else O.calib_absmax(g["x"], 0)
    assert np.array_equal(g["ax"], ax)
    aw = O.calib_absmax(g["W"], 1)
    assert np.array_equal(g["aw"], aw)
    s = O.smooth_factors(ax, aw, 0.5)
    assert np.array_equal(g["s"], s)
    wq, sw, gf, _ = O.fold_quant_weights(g["W"], s, g["gamma"] if ln else None)
    assert np.array_equal(g["wq"], wq) and np.array_equal(g["sw"], sw)
    xq, sx = O.ln_smooth_quant(g["x"], gamma_f=gf) if ln else O.ln_smooth_quant(g["x"], s=s)
    assert np.array_equal(g["xq"], xq) and np.array_equal(g["sx"], sx)
    rows = np.arange(M) if M <= 16 else np.linspace(0, M - 1, 9).astype(int)
    ref = O.w8a8_gemm(xq[rows], sx[rows], wq, sw, "bf16")
    assert assert_bf16_close(g["y"][rows], ref) == 1.0


SAMPLED = [(8192, 4096, 28672, True, 0.02), (2048, 14336, 4096, False, 0.02), (2048, 4096, 6144, True, 0.02),
           (2048, 12288, 36864, True, 0.015), (2048, 12288, 12288, False, 0.015),
           (2048, 12288, 49152, True, 0.015), (2048, 49152, 12288, False, 0.015), (16, 49152, 12288, False, 0.015)]


@pytest.mark.parametrize("M,K,N,ln,w_std", SAMPLED)
def test_large_layer_sampled_rows(M, K, N, ln, w_std):
    """Full-size prefill and 175B-class linears, calibrated on their own batch.  The statistics
    (activation absmax over all M rows, of LN(x) where a LayerNorm precedes; weight absmax), the
    smoothing factors, the folded LayerNorm weight, every weight code and every weight scale are
    compared with the oracle in full, bit for bit.  The per-token codes and scales, and the GEMM
    output, on sampled rows (every column of those rows) from the oracle's own chain."""
    g = _layer(M, K, N, 200 + M + N, w_std, ln)
    ax = O.calib_ln_absmax(g["x"], g["gamma"]) if ln else O.calib_absmax(g["x"], 0)
    assert np.array_equal(g["ax"], ax)
    aw = O.calib_absmax(g["W"], 1)
    assert np.array_equal(g["aw"], aw)
    s = O.smooth_factors(ax, aw, 0.5)
    assert np.array_equal(g["s"], s)
    wq, sw, gf, _ = O.fold_quant_weights(g["W"], s, g["gamma"] if ln else None)
    assert np.array_equal(g["sw"], sw)
    assert np.array_equal(g["wq"], wq)
    if ln:
        assert np.array_equal(g["gf"], gf)
    rows = np.unique(np.concatenate([np.linspace(0, M - 1, 6).astype(int), [M - 1]]))
    if ln:
        xq, sx = O.ln_smooth_quant(g["x"][rows], gamma_f=gf)
    else:
        xq, sx = O.ln_smooth_quant(g["x"][rows], s=s)
    assert np.array_equal(g["xq"][rows], xq) and np.array_equal(g["sx"][rows], sx)
    ref = O.w8a8_gemm(xq, sx, wq, sw, "bf16")
    assert assert_bf16_close(g["y"][rows], ref) == 1.0


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_long_plain_rows_divisors_outside_the_fast_range(dt):
    """Rows longer than 16384 in plain mode divide by s through a reciprocal; a segment with a
    factor outside [2^-90, 2^90] takes the correctly rounded division instead."""
    M, K = 9, 20480
    c = sq_inputs.make_case(M, K, 8, 77, x_dtype=dt, w_dtype=dt)
    s = np.exp(np.random.default_rng(5).uniform(-1, 3, K)).astype(np.float32)
    s[5] = np.float32(2.0 ** -100)   # first segment: huge quotients in channel 5
    s[4100] = np.float32(2.0 ** 95)  # second segment: tiny quotients in channel 4100
    xq, sx = sq.sq_ln_smooth_quant(dev(c.x), s=dev(s))
    r_xq, r_sx = O.ln_smooth_quant(c.x, s=s)
    assert np.array_equal(host(sx), r_sx)
    assert np.array_equal(host(xq), r_xq)


# ----------------------------------------------------------------------------- per-tensor granularity
@pytest.mark.parametrize("M,K", [(1, 16), (33, 256), (64, 4096), (9, 14336), (2, 49152), (300, 1040)])
@pytest.mark.parametrize("mode", ["ln", "plain"])
def test_per_tensor_dynamic(M, K, mode):
    c = sq_inputs.make_case(M, K, 8, 5 * M + K, beta_std=0.05)
    rng = np.random.default_rng(K + 2)
    s = np.exp(rng.uniform(-1, 3, K)).astype(np.float32)
    if mode == "ln":
        gf, bf = (c.gamma / s).astype(np.float32), (c.beta / s).astype(np.float32)
        xq, sx, sc = sq.sq_ln_smooth_quant_per_tensor(dev(c.x), gamma_f=dev(gf), beta_f=dev(bf))
        r_xq, r_sx, r_sc = O.ln_smooth_quant_per_tensor(c.x, gamma_f=gf, beta_f=bf)
    else:
        xq, sx, sc = sq.sq_ln_smooth_quant_per_tensor(dev(c.x), s=dev(s))
        r_xq, r_sx, r_sc = O.ln_smooth_quant_per_tensor(c.x, s=s)
    assert host(sc)[0] == np.float32(r_sc)
    assert np.array_equal(host(sx), r_sx)
    assert np.array_equal(host(xq), r_xq)


@pytest.mark.parametrize("K", [256, 4096, 14336, 49152])
@pytest.mark.parametrize("mode", ["ln", "plain"])
def test_per_tensor_static_clamps(K, mode):
    """A calibrated scale at half the batch's own: the largest values saturate at +-127."""
    M = 40
    c = sq_inputs.make_case(M, K, 8, K + 9)
    s = np.ones(K, np.float32)
    kw = dict(gamma_f=c.gamma) if mode == "ln" else dict(s=s)
    _, _, dyn = O.ln_smooth_quant_per_tensor(c.x, **kw)
    static = np.float32(dyn * 0.5)
    r_xq, r_sx, _ = O.ln_smooth_quant_per_tensor(c.x, static_scale=float(static), **kw)
    dkw = {k: dev(v) for k, v in kw.items()}
    xq, sx, sc = sq.sq_ln_smooth_quant_per_tensor(dev(c.x), scale=dev(np.array([static], np.float32)), static=True,
                                                  **dkw)
    assert np.array_equal(host(sx), r_sx) and host(sc)[0] == static
    assert np.array_equal(host(xq), r_xq)
    assert (np.abs(r_xq) == 127).sum() > 0


def test_per_tensor_linear_end_to_end():
    """Per-tensor activations through the GEMM: sx holds the one scale for every row."""
    c = sq_inputs.make_case(48, 512, 384, 77)
    W, x, g = dev(c.W), dev(c.x), dev(c.gamma)
    s = sq.sq_smooth_factors(sq.sq_calib_ln_absmax(x, g), sq.sq_calib_absmax(W, 1), 0.5)
    wq, sw, gf, _ = sq.sq_fold_quant_weights(W, s, g)
    xq, sx, _ = sq.sq_ln_smooth_quant_per_tensor(x, gamma_f=gf)
    y = sq.sq_w8a8_gemm(xq, sx, wq, sw)
    r_xq, r_sx, _ = O.ln_smooth_quant_per_tensor(c.x, gamma_f=host(gf))
    assert np.array_equal(host(xq), r_xq)
    assert assert_bf16_close(host(y), O.w8a8_gemm(r_xq, r_sx, host(wq), host(sw), "bf16")) == 1.0


# ----------------------------------------------------------------------------- smoothing folded into the previous linear
def test_next_smoothing_folded_into_previous_linear():
    """Linear A feeds linear B (no LayerNorm between); B's smoothing is folded into A's output
    scales, so A's GEMM emits B's smoothed input and B quantises it with unit factors.  Every
    intermediate matches the oracle's chain bit for bit."""
    rng = np.random.default_rng(12)
    M, K1, K2, N = 300, 1024, 512, 256
    x = (rng.standard_normal((M, K1)) * np.where(rng.random(K1) < 0.02, 40.0, 1.0)).astype(np.float32)
    WA = rng.normal(0, 0.03, (K1, K2)).astype(np.float32)
    WB = rng.normal(0, 0.03, (K2, N)).astype(np.float32)
    xd, WAd, WBd = dev(x), dev(WA), dev(WB)
    sA = sq.sq_smooth_factors(sq.sq_calib_absmax(xd, 0), sq.sq_calib_absmax(WAd, 1), 0.5)
    wqA, swA, _, _ = sq.sq_fold_quant_weights(WAd, sA)
    xqA, sxA = sq.sq_ln_smooth_quant(xd, s=sA)
    yA = sq.sq_w8a8_gemm(xqA, sxA, wqA, swA, out_dtype=torch.float32)
    sB = sq.sq_smooth_factors(sq.sq_calib_absmax(yA, 0), sq.sq_calib_absmax(WBd, 1), 0.5)
    wqB, swB, _, _ = sq.sq_fold_quant_weights(WBd, sB)
    swA2 = sq.sq_fold_next_smoothing(swA, sB)
    yA2 = sq.sq_w8a8_gemm(xqA, sxA, wqA, swA2, out_dtype=torch.float32)
    xqB, sxB = sq.sq_ln_smooth_quant(yA2, s=torch.ones(K2, dtype=torch.float32, device=DEV))
    yB = sq.sq_w8a8_gemm(xqB, sxB, wqB, swB, out_dtype=torch.float32)

    r_sA = O.smooth_factors(O.calib_absmax(x, 0), O.calib_absmax(WA, 1), 0.5)
    r_wqA, r_swA, _, _ = O.fold_quant_weights(WA, r_sA)
    r_xqA, r_sxA = O.ln_smooth_quant(x, s=r_sA)
    r_yA = O.w8a8_gemm(r_xqA, r_sxA, r_wqA, r_swA, "f32")
    r_sB = O.smooth_factors(O.calib_absmax(r_yA, 0), O.calib_absmax(WB, 1), 0.5)
    r_wqB, r_swB, _, _ = O.fold_quant_weights(WB, r_sB)
    r_swA2 = O.fold_next_smoothing(r_swA, r_sB)
    r_yA2 = O.w8a8_gemm(r_xqA, r_sxA, r_wqA, r_swA2, "f32")
    r_xqB, r_sxB = O.ln_smooth_quant(r_yA2, s=np.ones(K2, np.float32))
    r_yB = O.w8a8_gemm(r_xqB, r_sxB, r_wqB, r_swB, "f32")
    assert np.array_equal(host(sB), r_sB) and np.array_equal(host(swA2), r_swA2)
    assert np.array_equal(host(yA2), r_yA2)
    assert np.array_equal(host(xqB), r_xqB) and np.array_equal(host(sxB), r_sxB)
    assert np.array_equal(host(yB), r_yB)



# A full wave of CTA-pair tiles plus a short last wave: 2 x 38 = 76 tiles on 74 pairs, long K,
# so the last two tiles are split along K over the idle pairs and a second kernel sums the
# pieces.  Ragged last row tile (300 rows), column tile (9572 columns) and last K piece.
SPLIT_TAIL = (300, 9572, 16400)
SPLIT_ROWS = np.array([0, 1, 127, 128, 255, 256, 299])


def test_split_tail_gemm_sampled_rows():
    M, N, K = SPLIT_TAIL
    assert sq.sq_w8a8_gemm_workspace_size(M, N, K) > 0
    rng = np.random.default_rng(31)
    xq, wq = random_codes(rng, M, K, extreme_row=0), random_codes(rng, N, K)
    sx = rng.uniform(1e-3, 0.5, M).astype(np.float32)
    sw = rng.uniform(1e-5, 1e-2, N).astype(np.float32)
    dx, dw, dsx, dsw = dev(xq), dev(wq), dev(sx), dev(sw)
    ws = torch.zeros(sq.sq_w8a8_gemm_workspace_size(M, N, K), dtype=torch.uint8, device=DEV)
    acc = host(sq.sq_w8a8_gemm(dx, None, dw, None, out_dtype=torch.int32, workspace=ws))
    assert not ws.any()
    r = SPLIT_ROWS
    assert np.array_equal(acc[r], O.w8a8_gemm(xq[r], None, wq, None, "i32"))
    y, rmax = sq.sq_w8a8_gemm_rowmax(dx, dsx, dw, dsw, workspace=ws)
    assert not ws.any()
    ref = O.w8a8_gemm(xq[r], sx[r], wq, sw, "bf16")
    assert np.array_equal(host(y)[r], ref)
    assert np.array_equal(host(rmax)[r], O.calib_absmax(ref, 1))


def test_split_tail_is_optional():
    """The split tail needs a workspace; given none, the call runs the last tiles whole, with
    the same exact result."""
    M, N, K = SPLIT_TAIL
    rng = np.random.default_rng(17)
    xq, wq = random_codes(rng, M, K, extreme_row=0), random_codes(rng, N, K)
    dx, dw = dev(xq), dev(wq)
    with_ws = host(sq.sq_w8a8_gemm(dx, None, dw, None, out_dtype=torch.int32))
    without = torch.empty(M, N, dtype=torch.int32, device=DEV)
    f = sq.lib().sq_w8a8_gemm
    assert f(ctypes.c_void_p(dx.data_ptr()), None, ctypes.c_void_p(dw.data_ptr()), None, M, N, K,
             ctypes.c_void_p(without.data_ptr()), sq.SQ_I32, N, None, 0,
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    r = SPLIT_ROWS
    assert np.array_equal(with_ws, host(without))
    assert np.array_equal(with_ws[r], O.w8a8_gemm(xq[r], None, wq, None, "i32"))

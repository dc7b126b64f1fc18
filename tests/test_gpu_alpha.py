"""GPU parity of the migration-strength grid search against the oracle's search.

Every candidate's layer output is bit-identical on both sides (the INT8 path is exact); the
reference X_in W differs only by binary32 (GPU) versus binary64 (oracle) accumulation, which
moves each relative squared error by far less than 2e-3 of itself.  The chosen strength
must agree wherever the oracle's best and second-best errors differ by more than that."""
import numpy as np
import pytest
import torch

import oracle as O
import sq_inputs
import w8a8_smoothquant_gemm_b200 as sq

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def dev(a):
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).view(torch.bfloat16).to(DEV)
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.fixture(autouse=True)
def _no_device_error():
    sq.sq_device_error(clear=True)
    yield
    torch.cuda.synchronize()
    assert sq.sq_device_error(clear=True) == 0


CASES = [
    # M, K, N, layernorm, dtype, outlier multiplier
    (96, 256, 64, True, "bf16", 60.0),
    (300, 1024, 512, False, "bf16", 100.0),
    (1100, 4096, 384, True, "bf16", 100.0),
    (64, 512, 200, True, "f32", 30.0),
]


@pytest.mark.parametrize("M,K,N,ln,dt,mult", CASES)
def test_alpha_search_matches_oracle(M, K, N, ln, dt, mult):
    c = sq_inputs.make_case(M, K, N, M + K + N, x_dtype=dt, w_dtype=dt, outlier_mult=mult, beta_std=0.05)
    alphas = sq.alpha_grid(20)
    gamma = c.gamma if ln else None
    beta = c.beta if ln else None
    err, _ = sq.sq_alpha_search(dev(c.x), dev(c.W), alphas, gamma=dev(gamma), beta=dev(beta))
    got = err.cpu().numpy()
    ref = O.alpha_search(c.x, c.W, np.array(alphas, np.float32), gamma=gamma, beta=beta)
    assert np.all(np.abs(got - ref) <= 2e-3 * ref), np.max(np.abs(got - ref) / ref)
    order = np.argsort(ref)
    if ref[order[1]] - ref[order[0]] > 4e-3 * ref[order[0]]:
        assert int(np.argmin(got)) == int(order[0])


def test_alpha_search_single_strength_equals_the_layer():
    """One candidate: the search's error is the relative squared error of the library's own
    layer output against the reference product (computed here from the pieces)."""
    M, K, N = 128, 512, 256
    c = sq_inputs.make_case(M, K, N, 5)
    x, W, g = dev(c.x), dev(c.W), dev(c.gamma)
    err, _ = sq.sq_alpha_search(x, W, [0.5], gamma=g)
    s = sq.sq_smooth_factors(sq.sq_calib_ln_absmax(x, g), sq.sq_calib_absmax(W, 1), 0.5)
    wq, sw, gf, _ = sq.sq_fold_quant_weights(W, s, g)
    xq, sx = sq.sq_ln_smooth_quant(x, gamma_f=gf)
    yh = sq.sq_w8a8_gemm(xq, sx, wq, sw, out_dtype=torch.float32).double()
    Y = torch.from_numpy(O.layernorm(c.x, c.gamma).astype(np.float64) @ O.bf16_to_f32(c.W).astype(np.float64)).to(DEV)
    want = float(((yh - Y) ** 2).sum() / (Y ** 2).sum())
    assert abs(float(err[0]) - want) <= 2e-3 * want

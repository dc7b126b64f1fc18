"""The quotient behind every code: the library's shared-divisor division against IEEE division.

The demo page ("SmoothQuant大模型平滑量化技术", quantize_int8) defines a code as round(v / scale),
so the quotient must be the correctly rounded one.  The quantisers and the weight fold divide a
whole row (column) by one scale through a correctly rounded reciprocal and Markstein's correction
step.  Markstein's theorem makes that exact as long as no intermediate leaves the normal range;
these tests check it exhaustively where the kernels rely on it:
  * every divisor significand of the binade [1, 2), and of the two binades at the ends of the
    range where the kernels take the fast path (2^-90 and 2^89), against 256 (64 at the ends)
    dividends whose quotients cover 2^-12 .. 256 -- every magnitude that decides an INT8 or
    E4M3 code (|v / scale| <= 127 for a scale taken from the data's own absmax);
  * the device's IEEE division itself against the host's (numpy float32 division) on a random
    sample, so the reference of the exhaustive sweeps is pinned to an independent implementation.
"""
import numpy as np
import pytest
import torch

import w8a8_smoothquant_gemm_b200 as sq

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def binade(e: int, sign: float = 1.0) -> torch.Tensor:
    """All 2^23 binary32 values of [2^e, 2^(e+1)) (times sign) as a CUDA tensor."""
    bits = np.arange(1 << 23, dtype=np.uint32) + np.uint32((e + 127) << 23)
    v = bits.view(np.float32) * np.float32(sign)
    return torch.from_numpy(v).to(DEV)


def dividends(n: int, e_div: int, seed: int) -> torch.Tensor:
    """n dividends a = +-m 2^(e_div + k), m uniform in [1, 2) with random low bits, k in -11 .. 7, so
    that a / b for b in [2^e_div, 2^(e_div+1)) lies in 2^-12 .. 256."""
    rng = np.random.default_rng(seed)
    m = (np.uint32(127 << 23) | rng.integers(0, 1 << 23, n, dtype=np.uint32)).view(np.float32)
    k = rng.integers(-11, 8, n)
    sgn = np.where(rng.random(n) < 0.5, -1.0, 1.0)
    a = (m.astype(np.float64) * np.exp2(e_div + k) * sgn).astype(np.float32)
    # a few exact multiples and half-way multiples of small integers: quotients at and between codes
    a[:8] = np.float32(2.0 ** e_div) * np.array([1, 2.5, -3.5, 127, -127, 0.5, 63.5, 1.5], np.float32)
    return torch.from_numpy(a).to(DEV)


def run(a: torch.Tensor, b: torch.Tensor):
    counts, _ = sq.sq_selfcheck_shared_divisor(a, b)
    torch.cuda.synchronize()
    return [int(v) for v in counts.cpu()]


@pytest.mark.parametrize("sign", [1.0, -1.0])
def test_every_divisor_of_a_binade(sign):
    a = dividends(256, 0, 1)
    bad_scalar, bad_packed, checked = run(a, binade(0, sign))
    assert checked == 256 << 23
    assert bad_scalar == 0 and bad_packed == 0


@pytest.mark.parametrize("e", [-90, 89])
def test_binades_at_the_ends_of_the_fast_range(e):
    a = dividends(64, e, 200 + e)
    bad_scalar, bad_packed, checked = run(a, binade(e))
    assert checked == 64 << 23
    assert bad_scalar == 0 and bad_packed == 0


def test_outside_the_fast_range_and_zero_divisors():
    # divisors just outside [2^-90, 2^90] take the plain division; a zero divisor is skipped
    b = torch.tensor([2.0 ** -91, np.nextafter(np.float32(2.0 ** -90), np.float32(0)), 2.0 ** 91, 2.0 ** 100,
                      0.0], dtype=torch.float32, device=DEV)
    a = dividends(64, -30, 5)
    bad_scalar, bad_packed, checked = run(a, b)
    assert checked == 64 * 4 and bad_scalar == 0 and bad_packed == 0


def test_device_reference_matches_host_ieee_division():
    rng = np.random.default_rng(9)
    b = (rng.uniform(1.0, 2.0, 4096) * np.exp2(rng.integers(-4, 4, 4096)) *
         np.where(rng.random(4096) < 0.5, -1, 1)).astype(np.float32)
    a = (rng.uniform(0.5, 1.0, 512) * np.exp2(rng.integers(-6, 8, 512)) *
         np.where(rng.random(512) < 0.5, -1, 1)).astype(np.float32)
    bd, ad = torch.from_numpy(b).to(DEV), torch.from_numpy(a).to(DEV)
    counts, q = sq.sq_selfcheck_shared_divisor(ad, bd, want_quotients=True)
    host = (a[None, :] / b[:, None]).astype(np.float32)  # numpy float32 division: IEEE, nearest even
    assert np.abs(host).min() >= 2.0 ** -12 and np.abs(host).max() <= 2.0 ** 13
    got = q.cpu().numpy()
    # the scalar quotients the library uses equal the host's IEEE quotients bit for bit
    assert np.array_equal(got.view(np.uint32), host.view(np.uint32))
    assert [int(v) for v in counts.cpu()] == [0, 0, 4096 * 512]

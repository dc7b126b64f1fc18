// sq_codes.cu -- per-token INT8 codes of activations whose row maxima are already known.
//
// "4.2 W8A8 量化与 SmoothQuant", sec. 6: a linear's input comes from a LayerNorm or from the
// previous GEMM's output, and the smoothing diag(s)^-1 folds into that previous layer at no
// run-time cost ("量化：只压权重，与训练后量化（PTQ）", SmoothQuant section).  With the next
// linear's factors folded into this GEMM's output scales (sq_fold_next_smoothing), the GEMM
// emits the smoothed input y' = y / s_next itself, and its epilogue also takes the per-row max
// |y'| of the values it stores (sq_w8a8_gemm_rowmax).  What is left of the per-token quantiser
// is a codes pass: sx[m] = RN(rowmax[m] / 127), xq[m, j] = clamp(rne(y'[m, j] / sx[m]), -127, 127)
// -- the same arithmetic as sq_ln_smooth_quant in plain mode with unit factors (y' / 1 = y'),
// with one read of y' and no statistics pass.
#include <algorithm>

#include "sq_common.cuh"

namespace sqk {

constexpr int CODES_CHUNKS = 2;  // 8-element chunks per thread

// Block (b, m): chunks [b * 256 * CODES_CHUNKS, ...) of row m.
template <bool BF16>
__global__ void __launch_bounds__(256)
quant_codes_kernel(const char* __restrict__ x, int64_t K, int64_t ld_bytes, const float* __restrict__ rowmax,
                   int8_t* __restrict__ xq, float* __restrict__ sx) {
  allow_dependent_launch();
  const int64_t m = blockIdx.y;
  const float scale = __fdiv_rn(__ldg(rowmax + m), 127.0f);
  if (blockIdx.x == 0 && threadIdx.x == 0) sx[m] = scale;
  const SharedDivisor d(scale);
  const int64_t nchunks = K / 8;
  const char* row = x + m * ld_bytes;
  int8_t* qrow = xq + m * K;
  const int64_t c0 = (int64_t)blockIdx.x * 256 * CODES_CHUNKS + threadIdx.x;
  float f[CODES_CHUNKS][8];
#pragma unroll
  for (int i = 0; i < CODES_CHUNKS; ++i) {  // every load in flight before the first use
    const int64_t c = c0 + i * 256;
    if (c < nchunks) {
      if (BF16) {
        unpack8_bf16(ldg_stream16(row + c * 16), f[i]);
      } else {
        const uint4 a = ldg_stream16(row + c * 32), b = ldg_stream16(row + c * 32 + 16);
        f[i][0] = __uint_as_float(a.x); f[i][1] = __uint_as_float(a.y);
        f[i][2] = __uint_as_float(a.z); f[i][3] = __uint_as_float(a.w);
        f[i][4] = __uint_as_float(b.x); f[i][5] = __uint_as_float(b.y);
        f[i][6] = __uint_as_float(b.z); f[i][7] = __uint_as_float(b.w);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < CODES_CHUNKS; ++i) {
    const int64_t c = c0 + i * 256;
    if (c >= nchunks) continue;
    // the given max bounds every |y| of the row, so the quotient never leaves [-127, 127] up to
    // one rounding; the clamped form also covers a max taken from other data
    const uint2 w = d.fast ? pack8_codes<true, true>(f[i], d) : pack8_codes<false, true>(f[i], d);
    *reinterpret_cast<uint2*>(qrow + c * 8) = w;
  }
}

}  // namespace sqk

namespace sqh {

cudaError_t launch_quant_codes(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, const float* rowmax,
                               int8_t* xq, float* sx, cudaStream_t st) {
  const int64_t per_block = 256 * sqk::CODES_CHUNKS;
  const int64_t bx = (K / 8 + per_block - 1) / per_block;
  if (M > 65535) {  // one launch per 65535 rows (grid y limit)
    for (int64_t m0 = 0; m0 < M; m0 += 65535) {
      const int64_t rows = std::min<int64_t>(65535, M - m0);
      const cudaError_t e = launch_quant_codes((const char*)x + m0 * ldx * (bf16 ? 2 : 4), bf16, rows, K, ldx,
                                               rowmax + m0, xq + m0 * K, sx + m0, st);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  const dim3 grid((unsigned)bx, (unsigned)M);
  const int64_t ldb = ldx * (bf16 ? 2 : 4);
  if (bf16) sqk::quant_codes_kernel<true><<<grid, 256, 0, st>>>((const char*)x, K, ldb, rowmax, xq, sx);
  else sqk::quant_codes_kernel<false><<<grid, 256, 0, st>>>((const char*)x, K, ldb, rowmax, xq, sx);
  return cudaGetLastError();
}

}  // namespace sqh

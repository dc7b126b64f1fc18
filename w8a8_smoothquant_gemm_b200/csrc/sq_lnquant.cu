// sq_lnquant.cu -- fused LayerNorm -> X diag(s)^-1 -> per-token dynamic INT8.
//
// "4.2 W8A8 量化与 SmoothQuant", sec. 6: diag(s)^-1 is folded offline into LayerNorm's
// gamma and beta, so the runtime kernel is LayerNorm with gamma' = gamma/s, beta' = beta/s.
// Sec. 7.1 and "量化：只压权重，与训练后量化（PTQ）": activations are quantised per token,
// dynamically: sx_m = max_j |y_mj| / 127, xq = clamp(rne(y / sx_m), -127, 127).
// Without a preceding LayerNorm (input from a previous GEMM) y_j = x_j / s_j.
//
// One block of 256 threads per row, the row held in registers (one 16-byte vector per
// 8-element chunk), so the row crosses HBM once: read K * elt bytes, write K codes and
// one scale.  The LayerNorm statistics follow the fixed order of sq_rowln.cuh.
#include <algorithm>

#include "sq_rowln.cuh"

namespace sqk {

template <bool BF16, int MAXC, bool LN>
__global__ void __launch_bounds__(ROW_THREADS)
ln_smooth_quant_kernel(const char* __restrict__ x, int64_t M, int K, int64_t ld_bytes,
                       const float* __restrict__ gamma_f, const float* __restrict__ beta_f,
                       const float* __restrict__ s, float eps, int8_t* __restrict__ xq, float* __restrict__ sx) {
  __shared__ float red[3 * (ROW_WARPS + 1)];
  const int nchunks = K / 8;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    RowChunks<BF16, MAXC> rc;
    rc.load(x + m * ld_bytes, nchunks);
    float mu = 0.0f, rstd = 0.0f;
    if (LN) row_stats(rc, nchunks, K, eps, red, mu, rstd);
    // absmax of y
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = threadIdx.x + i * ROW_THREADS;
      if (c < nchunks) {
        float f[8], y[8];
        rc.get(i, f);
        if (LN) ln_chunk(f, mu, rstd, gamma_f, beta_f, c, y);
        else div_chunk(f, s, c, y);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(y[e]));
      }
    }
    amax = block_max(amax, red + 2 * (ROW_WARPS + 1));
    const float scale = __fdiv_rn(amax, 127.0f);
    if (threadIdx.x == 0) sx[m] = scale;
    int8_t* qrow = xq + m * (int64_t)K;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = threadIdx.x + i * ROW_THREADS;
      if (c < nchunks) {
        float f[8], y[8];
        rc.get(i, f);
        if (LN) ln_chunk(f, mu, rstd, gamma_f, beta_f, c, y);
        else div_chunk(f, s, c, y);
        uint2 packed;
        packed.x = pack4_s8(quant_code(y[0], scale), quant_code(y[1], scale), quant_code(y[2], scale),
                            quant_code(y[3], scale));
        packed.y = pack4_s8(quant_code(y[4], scale), quant_code(y[5], scale), quant_code(y[6], scale),
                            quant_code(y[7], scale));
        *reinterpret_cast<uint2*>(qrow + (int64_t)c * 8) = packed;
      }
    }
  }
}

}  // namespace sqk

namespace sqh {

template <bool BF16, int MAXC>
static cudaError_t launch_lnq_t(const void* x, int64_t M, int K, int64_t ld_bytes, const float* gamma_f,
                                const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                                cudaStream_t st) {
  const int64_t grid = std::min<int64_t>(M, (int64_t)num_sms() * 64);
  if (gamma_f)
    sqk::ln_smooth_quant_kernel<BF16, MAXC, true><<<(unsigned)grid, sqk::ROW_THREADS, 0, st>>>(
        (const char*)x, M, K, ld_bytes, gamma_f, beta_f, s, eps, xq, sx);
  else
    sqk::ln_smooth_quant_kernel<BF16, MAXC, false><<<(unsigned)grid, sqk::ROW_THREADS, 0, st>>>(
        (const char*)x, M, K, ld_bytes, gamma_f, beta_f, s, eps, xq, sx);
  return cudaGetLastError();
}

cudaError_t launch_ln_smooth_quant(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx,
                                   const float* gamma_f, const float* beta_f, const float* s, float eps,
                                   int8_t* xq, float* sx, cudaStream_t st) {
  const int64_t ldb = ldx * (bf16 ? 2 : 4);
  const int need = (int)((K / 8 + sqk::ROW_THREADS - 1) / sqk::ROW_THREADS);
  const int k = (int)K;
#define SQ_LNQ_CASE(C)                                                                                  \
  if (need <= C)                                                                                        \
    return bf16 ? launch_lnq_t<true, C>(x, M, k, ldb, gamma_f, beta_f, s, eps, xq, sx, st)              \
                : launch_lnq_t<false, (C > 16 ? 16 : C)>(x, M, k, ldb, gamma_f, beta_f, s, eps, xq, sx, st);
  SQ_LNQ_CASE(1) SQ_LNQ_CASE(2) SQ_LNQ_CASE(4) SQ_LNQ_CASE(8) SQ_LNQ_CASE(16) SQ_LNQ_CASE(24) SQ_LNQ_CASE(32)
#undef SQ_LNQ_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sqh

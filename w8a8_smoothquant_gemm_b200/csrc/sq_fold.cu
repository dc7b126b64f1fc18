// sq_fold.cu -- migration factors and the offline weight fold of SmoothQuant.
//
//   s_j = max|X_j|^alpha / max|W_j|^(1-alpha)          ("4.2 W8A8 量化与 SmoothQuant", sec. 4)
//   W' = diag(s) W, gamma' = gamma / s, beta' = beta / s  (sec. 6, LayerNorm folding)
//   sw_k = max_j |W'_jk| / 127, Wq[k, j] = clamp(rne(W'_jk / sw_k))   (sec. 7.1: weights
//   per output channel, static; "SmoothQuant大模型平滑量化技术" demo: max/127, round, clip)
//
// The fold kernel gives each block a strip of CW output channels (columns of W[K, N]).
// Pass 1 streams the strip once from HBM for the column max; pass 2 re-reads it (the
// strips resident at one time are sized to stay in L2) and writes the codes transposed
// through shared memory into Wq[N, K] (K contiguous), the GEMM's K-major operand.
#include <algorithm>

#include "sq_common.cuh"

namespace sqk {

__global__ void smooth_factors_kernel(const float* __restrict__ ax, const float* __restrict__ aw, int64_t K,
                                      float alpha, float* __restrict__ s) {
  const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= K) return;
  const double x = (double)ax[j];
  const double w = (double)aw[j];
  float r;
  if (!(x > 0.0) || !(w > 0.0)) {
    r = 1.0f;
  } else if (alpha == 0.5f) {
    r = __double2float_rn(__dsqrt_rn(__ddiv_rn(x, w)));
  } else if (alpha == 1.0f) {
    r = (float)x;
  } else if (alpha == 0.0f) {
    r = __double2float_rn(__ddiv_rn(1.0, w));
  } else {
    const double a = (double)alpha;
    const double t1 = __dmul_rn(a, log(x));
    const double t2 = __dmul_rn(__dsub_rn(1.0, a), log(w));
    r = __double2float_rn(exp(__dsub_rn(t1, t2)));
  }
  s[j] = r;
}

// Loads 8 consecutive W elements (one 16-byte vector for bf16, two for fp32) as fp32.
template <bool BF16>
__device__ __forceinline__ void load8(const char* p, float f[8]) {
  if (BF16) {
    unpack8_bf16(ldg_stream16(p), f);
  } else {
    const uint4 a = ldg_stream16(p), b = ldg_stream16(p + 16);
    f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y); f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
    f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y); f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
  }
}

// Block: 256 threads = (CW/8 column groups of 8) x (256 / (CW/8) row lanes).
// Pass-2 tile: TJ rows (j) x CW columns (k); codes staged transposed in shared memory as
// [CW][TJ + 16] bytes, then written as CW rows of TJ contiguous bytes of Wq.
template <bool BF16, int CW>
__global__ void __launch_bounds__(256)
fold_quant_kernel(const char* __restrict__ W, int64_t K, int64_t N, int64_t ldw_bytes,
                  const float* __restrict__ s, const float* __restrict__ gamma, const float* __restrict__ beta,
                  int8_t* __restrict__ Wq, float* __restrict__ sw, float* __restrict__ gamma_f,
                  float* __restrict__ beta_f) {
  constexpr int ELT = BF16 ? 2 : 4;
  constexpr int NG = CW / 8;           // column groups per strip
  constexpr int NR = 256 / NG;         // row lanes
  constexpr int TJ = NR > 64 ? NR : 64; // rows per pass-2 tile (every thread busy)
  constexpr int TPAD = TJ + 16;        // padded staging row (bytes), keeps 16-byte alignment
  __shared__ float red[NR][CW + 1];
  __shared__ float scale_s[CW];
  __shared__ __align__(16) int8_t stage[CW][TPAD];

  const int g = threadIdx.x % NG;      // column group
  const int rl = threadIdx.x / NG;     // row lane

  // gamma' and beta' (grid-stride over K)
  for (int64_t j = (int64_t)blockIdx.x * 256 + threadIdx.x; j < K; j += (int64_t)gridDim.x * 256) {
    const float sj = s[j];
    if (gamma && gamma_f) gamma_f[j] = __fdiv_rn(gamma[j], sj);
    if (beta && beta_f) beta_f[j] = __fdiv_rn(beta[j], sj);
  }

  const int64_t nstrips = (N + CW - 1) / CW;
  for (int64_t strip = blockIdx.x; strip < nstrips; strip += gridDim.x) {
    const int64_t k0 = strip * CW;
    const int64_t kc = k0 + g * 8;     // first column of this thread's group
    const bool col_ok = kc < N;        // N % 8 == 0, so a group is all in or all out
    // ---- pass 1: column max of |s_j * W[j, k]|
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = 0.0f;
    if (col_ok) {
      const char* colp = W + kc * ELT;
      int64_t j = rl;
      for (; j + 3 * NR < K; j += 4 * NR) {
        float f[4][8];
        float sj[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          load8<BF16>(colp + (j + u * NR) * ldw_bytes, f[u]);
          sj[u] = __ldg(s + j + u * NR);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(__fmul_rn(sj[u], f[u][e])));
      }
      for (; j < K; j += NR) {
        float f[8];
        load8<BF16>(colp + j * ldw_bytes, f);
        const float sj = __ldg(s + j);
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e] = fmaxf(m[e], fabsf(__fmul_rn(sj, f[e])));
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rl][g * 8 + e] = m[e];
    __syncthreads();
    if (threadIdx.x < CW) {
      float v = red[0][threadIdx.x];
      for (int r = 1; r < NR; ++r) v = fmaxf(v, red[r][threadIdx.x]);
      const float sc = __fdiv_rn(v, 127.0f);
      scale_s[threadIdx.x] = sc;
      if (k0 + threadIdx.x < N) sw[k0 + threadIdx.x] = sc;
    }
    __syncthreads();
    // ---- pass 2: codes, transposed through shared memory
    float sc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) sc[e] = scale_s[g * 8 + e];
    for (int64_t j0 = 0; j0 < K; j0 += TJ) {
      // each thread quantises 8 columns x (TJ / NR) rows of the tile
      for (int jj = rl; jj < TJ; jj += NR) {
        const int64_t j = j0 + jj;
        int q[8] = {0, 0, 0, 0, 0, 0, 0, 0};
        if (col_ok && j < K) {
          float f[8];
          load8<BF16>(W + j * ldw_bytes + kc * ELT, f);
          const float sj = __ldg(s + j);
#pragma unroll
          for (int e = 0; e < 8; ++e) q[e] = quant_code(__fmul_rn(sj, f[e]), sc[e]);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) stage[g * 8 + e][jj] = (int8_t)q[e];
      }
      __syncthreads();
      // write CW rows x TJ bytes: 4 x 16-byte pieces per row
      for (int t = threadIdx.x; t < CW * (TJ / 16); t += 256) {
        const int row = t / (TJ / 16), piece = t % (TJ / 16);
        const int64_t k = k0 + row;
        const int64_t j = j0 + piece * 16;
        if (k < N && j < K)  // K % 16 == 0: a piece is all in or all out
          *reinterpret_cast<uint4*>(Wq + k * K + j) = *reinterpret_cast<const uint4*>(&stage[row][piece * 16]);
      }
      __syncthreads();
    }
  }
}

}  // namespace sqk

namespace sqh {

cudaError_t launch_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s,
                                  cudaStream_t st) {
  const unsigned grid = (unsigned)((K + 255) / 256);
  sqk::smooth_factors_kernel<<<grid, 256, 0, st>>>(ax, aw, K, alpha, s);
  return cudaGetLastError();
}

template <bool BF16, int CW>
static cudaError_t launch_fold_t(const void* W, int64_t K, int64_t N, int64_t ldw, const float* s, const float* gamma,
                                 const float* beta, int8_t* Wq, float* sw, float* gamma_f, float* beta_f,
                                 cudaStream_t st) {
  const int64_t nstrips = (N + CW - 1) / CW;
  const int64_t elt = BF16 ? 2 : 4;
  // strips resident at once (one per block) should fit in about half of L2 so the
  // second pass hits L2: limit the grid accordingly, but keep at least one wave.
  int l2 = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&l2, cudaDevAttrL2CacheSize, dev);
  const int64_t strip_bytes = K * CW * elt;
  int64_t fit = std::max<int64_t>(1, (int64_t)l2 / 2 / std::max<int64_t>(strip_bytes, 1));
  int64_t grid = std::min<int64_t>(nstrips, std::max<int64_t>(std::min<int64_t>(fit, (int64_t)num_sms() * 4),
                                                              (int64_t)num_sms()));
  grid = std::max<int64_t>(grid, 1);
  sqk::fold_quant_kernel<BF16, CW><<<(unsigned)grid, 256, 0, st>>>((const char*)W, K, N, ldw * elt, s, gamma, beta,
                                                                   Wq, sw, gamma_f, beta_f);
  return cudaGetLastError();
}

cudaError_t launch_fold_quant(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw, const float* s,
                              const float* gamma, const float* beta, int8_t* Wq, float* sw, float* gamma_f,
                              float* beta_f, cudaStream_t st) {
  // narrower strips when there are few output channels, so every SM gets work
  const int64_t sms = num_sms();
  const int cw = (N / 32 >= 2 * sms) ? 32 : 16;
  if (bf16)
    return cw == 32 ? launch_fold_t<true, 32>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st)
                    : launch_fold_t<true, 16>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
  return cw == 32 ? launch_fold_t<false, 32>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st)
                  : launch_fold_t<false, 16>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
}

}  // namespace sqh

// sq_fold.cu -- migration factors and the offline weight fold of SmoothQuant.
//
//   s_j = max|X_j|^alpha / max|W_j|^(1-alpha)          ("4.2 W8A8 量化与 SmoothQuant", sec. 4)
//   W' = diag(s) W, gamma' = gamma / s, beta' = beta / s  (sec. 6, LayerNorm folding)
//   sw_k = max_j |W'_jk| / 127, Wq[k, j] = clamp(rne(W'_jk / sw_k))   (sec. 7.1: weights
//   per output channel, static; "SmoothQuant大模型平滑量化技术" demo: max/127, round, clip)
//
// Wq is written transposed, [N, K] with K contiguous: the GEMM's K-major operand.  Three
// routes cover the shapes:
//   fold_cluster_kernel  bf16 W of at most 96 MiB whose K / 16 rows per CTA fit 72 KB of
//                        shared memory: one pass over HBM, column maxima exchanged in a
//                        thread-block cluster;
//   streaming fold       larger or taller bf16 W: fold_colmax_kernel (column maxima), then
//                        fold_codes_stream_kernel (codes of TMA-loaded tiles, last rows
//                        first so that the part of W still in L2 is reused), then
//                        fold_scales_kernel;
//   fold_quant_kernel    fp32 or unaligned W: one block per strip, two passes.
#include <algorithm>

#include "sq_ptx.cuh"

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

// sw'[n] = RN(sw[n] / s_next[n]): the next linear's smoothing diag(s_next)^-1 folded into this
// linear's per-output-channel scale ("量化：只压权重…", SmoothQuant section: diag(s)^-1 folds
// offline into the preceding LayerNorm or linear layer), so this layer's output is already
// the smoothed input of the next one.
__global__ void fold_next_smoothing_kernel(const float* __restrict__ sw, const float* __restrict__ s_next, int64_t N,
                                           float* __restrict__ out) {
  const int64_t n = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (n < N) out[n] = __fdiv_rn(sw[n], s_next[n]);
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
template <bool BF16, int CW, bool F8>
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
      const float sc = __fdiv_rn(v, F8 ? 448.0f : 127.0f);
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
          for (int e = 0; e < 8; ++e) q[e] = F8 ? e4m3_code(__fmul_rn(sj, f[e]), sc[e]) : quant_code(__fmul_rn(sj, f[e]), sc[e]);
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

// ---------------------------------------------------------------------------- cluster fold
// One thread-block cluster of C CTAs per strip of CW output channels.  CTA r of the
// cluster owns rows [r * RK, (r + 1) * RK) of W (input channels): one thread TMA-loads that
// RK x CW block into shared memory in 64-row pieces, each completing on its own mbarrier,
// so the column-max pass follows the data in (W crosses HBM once).  Each CTA pushes its
// partial column maxima of |s_j W_jk| into every peer's shared memory (distributed shared
// memory), one cluster barrier later every CTA has all C partials, and it quantises its
// block from shared memory, writing Wq[k, j] transposed, 16 codes at a time.  Rows beyond
// K and columns beyond N are zero-filled by TMA and never stored.
// Codes of a 16-row x 4-column block of the staged tile (rows jl.., columns kq..kq+3),
// as 4 words per column; FAST selects the Markstein-only division.
template <bool FAST>
__device__ __forceinline__ void fold_codes_16x4(const uint16_t* tile, const float* s_rows, int cw, int jl, int kq,
                                                const SharedDivisor& d0, const SharedDivisor& d1,
                                                const SharedDivisor& d2, const SharedDivisor& d3,
                                                uint32_t (&words)[4][4]) {
  // two adjacent columns per packed binary32 pair, each with its own scale; each half
  // rounds as the scalar operation would
  const float2 rc01 = make_float2(d0.y, d1.y), rc23 = make_float2(d2.y, d3.y);
  const float2 nb01 = make_float2(-d0.b, -d1.b), nb23 = make_float2(-d2.b, -d3.b);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4) {
    uint32_t b[4][4];
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = jl + g4 * 4 + r;
      const uint2 w = *reinterpret_cast<const uint2*>(tile + j * cw + kq);
      const float sj = s_rows[j];
      const float2 y01 = __fmul2_rn(make_float2(sj, sj), make_float2(bf16lo(w.x), bf16hi(w.x)));
      const float2 y23 = __fmul2_rn(make_float2(sj, sj), make_float2(bf16lo(w.y), bf16hi(w.y)));
      if (FAST) {
        const float2 t01 = __fadd2_rn(markstein2(y01, rc01, nb01), magic);
        const float2 t23 = __fadd2_rn(markstein2(y23, rc23, nb23), magic);
        b[0][r] = __float_as_uint(t01.x);
        b[1][r] = __float_as_uint(t01.y);
        b[2][r] = __float_as_uint(t23.x);
        b[3][r] = __float_as_uint(t23.y);
      } else {
        b[0][r] = code_bits(y01.x, d0);
        b[1][r] = code_bits(y01.y, d1);
        b[2][r] = code_bits(y23.x, d2);
        b[3][r] = code_bits(y23.y, d3);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) words[c][g4] = pack4_low_bytes(b[c][0], b[c][1], b[c][2], b[c][3]);
  }
}

// E4M3 codes of a 16-row x 4-column block (the FP8 variant): the quotients of
// fold_codes_16x4 with the dividend's sign kept on zero results (Markstein's correction
// turns RN(-0 / b) into +0), converted with saturation; a zero scale gives +0 codes.
// FAST: every scale nonzero and in Markstein's range.
template <bool FAST>
__device__ __forceinline__ void fold_codes_16x4_e4m3(const uint16_t* tile, const float* s_rows, int cw, int jl, int kq,
                                                     const SharedDivisor& d0, const SharedDivisor& d1,
                                                     const SharedDivisor& d2, const SharedDivisor& d3,
                                                     uint32_t (&words)[4][4]) {
  const float2 rc01 = make_float2(d0.y, d1.y), rc23 = make_float2(d2.y, d3.y);
  const float2 nb01 = make_float2(-d0.b, -d1.b), nb23 = make_float2(-d2.b, -d3.b);
  const SharedDivisor* dv[4] = {&d0, &d1, &d2, &d3};
#pragma unroll
  for (int g4 = 0; g4 < 4; ++g4) {
    float q[4][4];  // [column][row]
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const int j = jl + g4 * 4 + r;
      const uint2 w = *reinterpret_cast<const uint2*>(tile + j * cw + kq);
      const float sj = s_rows[j];
      const float2 y01 = __fmul2_rn(make_float2(sj, sj), make_float2(bf16lo(w.x), bf16hi(w.x)));
      const float2 y23 = __fmul2_rn(make_float2(sj, sj), make_float2(bf16lo(w.y), bf16hi(w.y)));
      if (FAST) {
        const float2 t01 = markstein2(y01, rc01, nb01);
        const float2 t23 = markstein2(y23, rc23, nb23);
        q[0][r] = with_sign_of(t01.x, y01.x);
        q[1][r] = with_sign_of(t01.y, y01.y);
        q[2][r] = with_sign_of(t23.x, y23.x);
        q[3][r] = with_sign_of(t23.y, y23.y);
      } else {
        const float y[4] = {y01.x, y01.y, y23.x, y23.y};
#pragma unroll
        for (int c = 0; c < 4; ++c)
          q[c][r] = (dv[c]->fast && dv[c]->y == 0.0f) ? 0.0f : with_sign_of(dv[c]->div(y[c]), y[c]);
      }
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) words[c][g4] = e4m3x4(q[c][0], q[c][1], q[c][2], q[c][3]);
  }
}

// Codes of this CTA's rows of the strip at column k0 from the staged tile, with the
// strip's scales, written to Wq transposed: item = (4 adjacent columns, 16 consecutive
// rows); each item reads 16 x 8 bytes of shared memory and writes 16 codes to each of 4
// rows of Wq.  F8: E4M3 codes (the FP8 variant).
template <int CW, bool F8, int NT = 256>
__device__ __forceinline__ void fold_write_codes(const uint16_t* tile, const float* s_rows, const float* scale,
                                                 int64_t K, int64_t N, int RK, int64_t j0, int64_t k0,
                                                 int8_t* __restrict__ Wq) {
  const int items = (CW / 4) * (RK / 16);
  for (int i = threadIdx.x; i < items; i += NT) {
    const int kq = (i % (CW / 4)) * 4, jl = (i / (CW / 4)) * 16;
    if (j0 + jl >= K) continue;  // K % 16 == 0: a 16-row block is all in or all out
    const SharedDivisor d0(scale[kq]), d1(scale[kq + 1]), d2(scale[kq + 2]), d3(scale[kq + 3]);
    uint32_t words[4][4];
    const bool fast = d0.fast && d1.fast && d2.fast && d3.fast;
    if (F8) {
      if (fast && d0.y != 0.0f && d1.y != 0.0f && d2.y != 0.0f && d3.y != 0.0f)
        fold_codes_16x4_e4m3<true>(tile, s_rows, CW, jl, kq, d0, d1, d2, d3, words);
      else
        fold_codes_16x4_e4m3<false>(tile, s_rows, CW, jl, kq, d0, d1, d2, d3, words);
    } else if (fast) {
      fold_codes_16x4<true>(tile, s_rows, CW, jl, kq, d0, d1, d2, d3, words);
    } else {
      fold_codes_16x4<false>(tile, s_rows, CW, jl, kq, d0, d1, d2, d3, words);
    }
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int64_t k = k0 + kq + c;
      if (k < N)
        *reinterpret_cast<uint4*>(Wq + k * K + j0 + jl) = make_uint4(words[c][0], words[c][1], words[c][2], words[c][3]);
    }
  }
}

constexpr int FOLD_MAX_CLUSTER = 16;
constexpr int FOLD_MAX_PIECES = 64;  // RK <= 4096 rows per CTA

template <int CW, bool F8>
__global__ void __launch_bounds__(256)
fold_cluster_kernel(const __grid_constant__ CUtensorMap wmap, int64_t K, int64_t N, int RK, int C,
                    const float* __restrict__ s, const float* __restrict__ gamma, const float* __restrict__ beta,
                    int8_t* __restrict__ Wq, float* __restrict__ sw, float* __restrict__ gamma_f,
                    float* __restrict__ beta_f, unsigned int* err) {
  constexpr int G = 256 / (CW / 8);  // row lanes of the max pass (8 columns per thread)
  extern __shared__ uint8_t smem_raw[];
  // TMA destinations want 128-byte alignment: round the dynamic base up (128 bytes of slack)
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const uint16_t* tile = reinterpret_cast<const uint16_t*>(smem);      // [RK][CW] bf16 bits
  float* s_rows = reinterpret_cast<float*>(smem + (size_t)RK * CW * 2);  // [RK]
  __shared__ float red[G][CW + 1];
  __shared__ float part[FOLD_MAX_CLUSTER][CW];  // partial maxima of every CTA of the cluster
  __shared__ float scale[CW];
  __shared__ __align__(8) uint64_t bars[FOLD_MAX_PIECES];

  const int tid = threadIdx.x;
  const uint32_t crank = cluster_ctarank();
  const unsigned long long limit = wait_limit(err);
  const int64_t strip = blockIdx.x / C;
  const int64_t k0 = strip * CW;
  const int64_t j0 = (int64_t)crank * RK;
  const int pieces = RK / 64;

  for (int64_t j = (int64_t)blockIdx.x * 256 + tid; j < K; j += (int64_t)gridDim.x * 256) {
    const float sj = s[j];
    if (gamma && gamma_f) gamma_f[j] = __fdiv_rn(gamma[j], sj);
    if (beta && beta_f) beta_f[j] = __fdiv_rn(beta[j], sj);
  }

  if (tid == 0) {
    for (int p = 0; p < pieces; ++p) mbar_init(smem_u32(&bars[p]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0) {
    for (int p = 0; p < pieces; ++p) {
      const uint32_t b = smem_u32(&bars[p]);
      mbar_arrive_expect_tx(b, (uint32_t)64 * CW * 2);
      tma_load_2d(smem_u32(smem + (size_t)p * 64 * CW * 2), &wmap, b, (int)k0, (int)(j0 + p * 64));
    }
  }
  for (int i = tid; i < RK; i += 256) s_rows[i] = (j0 + i < K) ? __ldg(s + j0 + i) : 0.0f;
  __syncthreads();

  // ---- partial column max of |s_j W_jk| over this CTA's rows, piece by piece as they land:
  // thread = 8 columns x rows rl, rl + G, ...
  bool failed = false;
  {
    const int cg = tid % (CW / 8), rl = tid / (CW / 8);
    float m[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) m[e] = 0.0f;
    for (int p = 0; p < pieces; ++p) {
      if (!mbar_wait(smem_u32(&bars[p]), 0, limit)) {
        failed = true;  // stop reading this block; the cluster exchange below still takes place
        break;
      }
      for (int j = p * 64 + rl; j < p * 64 + 64; j += G) {
        const uint4 w = *reinterpret_cast<const uint4*>(tile + j * CW + cg * 8);
        const float2 sj = make_float2(s_rows[j], s_rows[j]);
        const float2 y0 = __fmul2_rn(sj, make_float2(bf16lo(w.x), bf16hi(w.x)));
        const float2 y1 = __fmul2_rn(sj, make_float2(bf16lo(w.y), bf16hi(w.y)));
        const float2 y2 = __fmul2_rn(sj, make_float2(bf16lo(w.z), bf16hi(w.z)));
        const float2 y3 = __fmul2_rn(sj, make_float2(bf16lo(w.w), bf16hi(w.w)));
        m[0] = fmaxf(m[0], fabsf(y0.x)); m[1] = fmaxf(m[1], fabsf(y0.y));
        m[2] = fmaxf(m[2], fabsf(y1.x)); m[3] = fmaxf(m[3], fabsf(y1.y));
        m[4] = fmaxf(m[4], fabsf(y2.x)); m[5] = fmaxf(m[5], fabsf(y2.y));
        m[6] = fmaxf(m[6], fabsf(y3.x)); m[7] = fmaxf(m[7], fabsf(y3.y));
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[rl][cg * 8 + e] = m[e];
  }
  failed = __syncthreads_or(failed);
  if (failed && tid == 0) {
    atomicOr(err, ERR_FOLD_TMA_WAIT);
    for (int p = 0; p < pieces; ++p) (void)mbar_wait(smem_u32(&bars[p]), 0, DRAIN_NS);  // issued copies land
  }
  if (tid < CW) {
    float m = red[0][tid];
    for (int g = 1; g < G; ++g) m = fmaxf(m, red[g][tid]);
    for (int r = 0; r < C; ++r) st_dsmem_f32(&part[crank][tid], (uint32_t)r, m);  // into every CTA
  }
  cluster_sync();  // all partials delivered; no CTA touches a peer's memory after this
  if (tid < CW) {
    float m = 0.0f;
    for (int r = 0; r < C; ++r) m = fmaxf(m, part[r][tid]);
    const float sc = __fdiv_rn(m, F8 ? 448.0f : 127.0f);
    scale[tid] = sc;
    if (crank == 0 && k0 + tid < N) sw[k0 + tid] = sc;
  }
  __syncthreads();

  // ---- codes, transposed (not after a wait ran out: the block's data is incomplete)
  if (!failed) fold_write_codes<CW, F8>(tile, s_rows, scale, K, N, RK, j0, k0, Wq);
}

// ---------------------------------------------------------------------------- two-pass fold
// Pass 1 of the streaming fold: column maxima of |s_j W_jk| over all rows.  A block is 32
// 16-byte column vectors x 8 row lanes; the grid covers the columns once and strides the
// rows with four loads in flight per thread, so the loads of all blocks sweep W from the
// first rows to the last; one atomicMax per column per block into colmax (zeroed before).
// Also writes the folded LayerNorm vectors gamma' = gamma / s, beta' = beta / s.
constexpr int FCM_VX = 32, FCM_RY = 8, FCM_UNROLL = 4;

__device__ __forceinline__ void colmax8(float (&m)[8], const uint4 v, float sj) {
  const float2 s2 = make_float2(sj, sj);
  const float2 y0 = __fmul2_rn(s2, make_float2(bf16lo(v.x), bf16hi(v.x)));
  const float2 y1 = __fmul2_rn(s2, make_float2(bf16lo(v.y), bf16hi(v.y)));
  const float2 y2 = __fmul2_rn(s2, make_float2(bf16lo(v.z), bf16hi(v.z)));
  const float2 y3 = __fmul2_rn(s2, make_float2(bf16lo(v.w), bf16hi(v.w)));
  m[0] = fmaxf(m[0], fabsf(y0.x)); m[1] = fmaxf(m[1], fabsf(y0.y));
  m[2] = fmaxf(m[2], fabsf(y1.x)); m[3] = fmaxf(m[3], fabsf(y1.y));
  m[4] = fmaxf(m[4], fabsf(y2.x)); m[5] = fmaxf(m[5], fabsf(y2.y));
  m[6] = fmaxf(m[6], fabsf(y3.x)); m[7] = fmaxf(m[7], fabsf(y3.y));
}

__global__ void __launch_bounds__(FCM_VX * FCM_RY)
fold_colmax_kernel(const char* __restrict__ W, int64_t K, int64_t nvec, int64_t ldw_bytes,
                   const float* __restrict__ s, float* __restrict__ colmax, const float* __restrict__ gamma,
                   const float* __restrict__ beta, float* __restrict__ gamma_f, float* __restrict__ beta_f) {
  __shared__ float red[FCM_RY][FCM_VX * 8 + 1];
  const int tid = threadIdx.y * FCM_VX + threadIdx.x;
  if (gamma_f || beta_f) {
    const int64_t nb = (int64_t)gridDim.x * gridDim.y, b = (int64_t)blockIdx.y * gridDim.x + blockIdx.x;
    for (int64_t j = b * 256 + tid; j < K; j += nb * 256) {
      const float sj = s[j];
      if (gamma && gamma_f) gamma_f[j] = __fdiv_rn(gamma[j], sj);
      if (beta && beta_f) beta_f[j] = __fdiv_rn(beta[j], sj);
    }
  }
  const int64_t vec = (int64_t)blockIdx.x * FCM_VX + threadIdx.x;
  float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (vec < nvec) {
    const int64_t rstep = (int64_t)gridDim.y * FCM_RY;
    int64_t r = (int64_t)blockIdx.y * FCM_RY + threadIdx.y;
    const char* p = W + vec * 16;
    for (; r + (FCM_UNROLL - 1) * rstep < K; r += FCM_UNROLL * rstep) {
      uint4 v[FCM_UNROLL];
      float sj[FCM_UNROLL];
#pragma unroll
      for (int u = 0; u < FCM_UNROLL; ++u) {
        v[u] = ldg_stream16(p + (r + u * rstep) * ldw_bytes);
        sj[u] = __ldg(s + r + u * rstep);
      }
#pragma unroll
      for (int u = 0; u < FCM_UNROLL; ++u) colmax8(m, v[u], sj[u]);
    }
    for (; r < K; r += rstep) colmax8(m, ldg_stream16(p + r * ldw_bytes), __ldg(s + r));
  }
#pragma unroll
  for (int e = 0; e < 8; ++e) red[threadIdx.y][threadIdx.x * 8 + e] = m[e];
  __syncthreads();
  const int64_t ncols = nvec * 8;
  for (int c = tid; c < FCM_VX * 8; c += FCM_VX * FCM_RY) {
    float v = red[0][c];
#pragma unroll
    for (int y = 1; y < FCM_RY; ++y) v = fmaxf(v, red[y][c]);
    const int64_t col = (int64_t)blockIdx.x * FCM_VX * 8 + c;
    if (col < ncols) atomic_max_nonneg(colmax + col, v);
  }
}

// Pass 2: the codes of RT-row x 64-column tiles of W (RT threads, one 16-row x 4-column item
// each), written transposed into Wq (fold_write_codes).  Persistent blocks walk the tiles
// with the last rows first: pass 1 read those last, so the part of W still in L2 is read
// from there.  One thread TMA-loads each tile into an S-stage shared-memory ring, S - 1
// tiles ahead of the block's codes.
constexpr int FCS_CW = 64;

template <int RT, int S, bool F8>
__global__ void __launch_bounds__(RT, 896 / RT)  // 7 blocks of 128 threads per SM (72 registers)
fold_codes_stream_kernel(const __grid_constant__ CUtensorMap wmap, int64_t K, int64_t N,
                         const float* __restrict__ s, const float* __restrict__ colmax, int8_t* __restrict__ Wq,
                         unsigned int* err) {
  constexpr uint32_t TILE = RT * FCS_CW * 2;
  static_assert(RT >= FCS_CW && (FCS_CW / 4) * (RT / 16) == RT, "one item per thread");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  __shared__ float s_rows[RT];
  __shared__ float scale[FCS_CW];
  __shared__ __align__(8) uint64_t bars[S];
  const int tid = threadIdx.x;
  const unsigned long long limit = wait_limit(err);
  const int64_t strips = (N + FCS_CW - 1) / FCS_CW, rtiles = (K + RT - 1) / RT;
  const int64_t units = strips * rtiles;
  const int64_t first = blockIdx.x, step = gridDim.x;
  auto row0 = [&](int64_t u) { return (rtiles - 1 - u / strips) * RT; };
  auto col0 = [&](int64_t u) { return (u % strips) * FCS_CW; };
  auto issue = [&](int64_t u, int stage) {
    const uint32_t b = smem_u32(&bars[stage]);
    mbar_arrive_expect_tx(b, TILE);
    tma_load_2d(smem_u32(ring + (size_t)stage * TILE), &wmap, b, (int)col0(u), (int)row0(u));
  };
  if (tid == 0) {
    for (int i = 0; i < S; ++i) mbar_init(smem_u32(&bars[i]), 1);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0)
    for (int i = 0; i < S - 1 && first + i * step < units; ++i) issue(first + i * step, i);
  for (int64_t i = 0; first + i * step < units; ++i) {
    const int64_t u = first + i * step;
    const int64_t j0 = row0(u), k0 = col0(u);
    // the stage of tile i + S - 1 held tile i - 1, whose reads ended at the previous barrier
    if (tid == 0 && u + (S - 1) * step < units) {
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      issue(u + (S - 1) * step, (int)((i + S - 1) % S));
    }
    s_rows[tid] = (j0 + tid < K) ? __ldg(s + j0 + tid) : 0.0f;
    if (tid < FCS_CW) scale[tid] = (k0 + tid < N) ? __fdiv_rn(__ldg(colmax + k0 + tid), F8 ? 448.0f : 127.0f) : 0.0f;
    __syncthreads();
    const int stage = (int)(i % S);
    const bool ok = mbar_wait(smem_u32(&bars[stage]), (uint32_t)((i / S) & 1), limit);
    if (__syncthreads_or(!ok)) {
      // the block stops: the tiles it has issued (i .. i + S - 1) land before it leaves
      if (tid == 0) {
        atomicOr(err, ERR_FOLD_TMA_WAIT);
        for (int j = 0; j < S; ++j)
          if (first + (i + j) * step < units)
            (void)mbar_wait(smem_u32(&bars[(int)((i + j) % S)]), (uint32_t)(((i + j) / S) & 1), DRAIN_NS);
      }
      break;
    }
    fold_write_codes<FCS_CW, F8, RT>(reinterpret_cast<const uint16_t*>(ring + (size_t)stage * TILE), s_rows, scale,
                                     K, N, RT, j0, k0, Wq);
    __syncthreads();
  }
}

// sw[k] = RN(max_k / 127) (F8: / 448) in place.
template <bool F8>
__global__ void fold_scales_kernel(float* __restrict__ sw, int64_t N) {
  const int64_t k = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (k < N) sw[k] = __fdiv_rn(sw[k], F8 ? 448.0f : 127.0f);
}
}  // namespace sqk


namespace sqh {

cudaError_t launch_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s,
                                  cudaStream_t st) {
  const unsigned grid = (unsigned)((K + 255) / 256);
  sqk::smooth_factors_kernel<<<grid, 256, 0, st>>>(ax, aw, K, alpha, s);
  return cudaGetLastError();
}

cudaError_t launch_fold_next_smoothing(const float* sw, const float* s_next, int64_t N, float* out, cudaStream_t st) {
  sqk::fold_next_smoothing_kernel<<<(unsigned)((N + 255) / 256), 256, 0, st>>>(sw, s_next, N, out);
  return cudaGetLastError();
}

template <bool BF16, int CW, bool F8>
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
  sqk::fold_quant_kernel<BF16, CW, F8><<<(unsigned)grid, 256, 0, st>>>((const char*)W, K, N, ldw * elt, s, gamma, beta,
                                                                   Wq, sw, gamma_f, beta_f);
  return cudaGetLastError();
}

template <int CW, bool F8>
static cudaError_t launch_fold_cluster_t(const void* W, int64_t K, int64_t N, int64_t ldw, int C, int RK,
                                         const float* s, const float* gamma, const float* beta, int8_t* Wq,
                                         float* sw, float* gamma_f, float* beta_f, cudaStream_t st) {
  CUtensorMap map;
  if (!make_tmap_2d(&map, true, W, N, K, ldw * 2, CW, 64, false)) return cudaErrorInvalidValue;
  const size_t smem = 128 + (size_t)RK * CW * 2 + (size_t)RK * 4;
  auto kern = sqk::fold_cluster_kernel<CW, F8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if (C > 8) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  const int64_t strips = (N + CW - 1) / CW;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(strips * C));
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, map, K, N, RK, C, s, gamma, beta, Wq, sw, gamma_f, beta_f, error_word_ptr());
}

// Cluster shape of the single-pass fold: C CTAs share a strip (at least 256 rows each, at
// most 16), and the strip is the widest CW whose per-CTA block fits `budget` bytes of
// shared memory.
static bool fold_cluster_shape(int64_t K, size_t budget, int* cw, int* c, int* rk) {
  const int cl = (int)std::min<int64_t>(16, std::max<int64_t>(1, (K + 255) / 256));
  const int64_t rows = ((K + cl - 1) / cl + 63) / 64 * 64;
  if (rows / 64 > sqk::FOLD_MAX_PIECES) return false;
  for (int w : {64, 32, 16})
    if ((size_t)rows * w * 2 + (size_t)rows * 4 <= budget) {
      *cw = w;
      *c = cl;
      *rk = (int)rows;
      return true;
    }
  return false;
}

// Streaming two-pass fold of bf16 weights: column maxima into sw, the codes pass (RT-row
// tiles in an S-stage TMA ring, as many blocks as fit on the SMs), then the maxima in sw
// become scales.
template <int RT, int S, bool F8>
static cudaError_t launch_fold_stream(const void* W, int64_t K, int64_t N, int64_t ldw, const float* s,
                                      const float* gamma, const float* beta, int8_t* Wq, float* sw, float* gamma_f,
                                      float* beta_f, cudaStream_t st) {
  CUtensorMap map;
  if (!make_tmap_2d(&map, true, W, N, K, ldw * 2, sqk::FCS_CW, RT, false)) return cudaErrorInvalidValue;
  cudaError_t e = cudaMemsetAsync(sw, 0, sizeof(float) * (size_t)N, st);
  if (e != cudaSuccess) return e;
  const int64_t nvec = N / 8;
  const int64_t gx = (nvec + sqk::FCM_VX - 1) / sqk::FCM_VX;
  // one wave: as many blocks as are resident at once (44 registers: 5 per SM), each
  // striding over the rows; measured 114 against 119 us at 4096 x 28672 over 8 per SM
  int occ = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, sqk::fold_colmax_kernel, sqk::FCM_VX * sqk::FCM_RY, 0);
  if (e != cudaSuccess) return e;
  int64_t gy = std::max<int64_t>(1, (int64_t)num_sms() * std::max(occ, 1) / gx);
  gy = std::min<int64_t>(gy, (K + sqk::FCM_RY - 1) / sqk::FCM_RY);
  gy = std::min<int64_t>(gy, 65535);
  sqk::fold_colmax_kernel<<<dim3((unsigned)gx, (unsigned)gy), dim3(sqk::FCM_VX, sqk::FCM_RY), 0, st>>>(
      (const char*)W, K, nvec, ldw * 2, s, sw, gamma, beta, gamma_f, beta_f);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  auto kern = sqk::fold_codes_stream_kernel<RT, S, F8>;
  const size_t smem = 128 + (size_t)S * RT * sqk::FCS_CW * 2;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, RT, smem);
  if (e != cudaSuccess) return e;
  const int64_t units = (N + sqk::FCS_CW - 1) / sqk::FCS_CW * ((K + RT - 1) / RT);
  const int64_t grid = std::min<int64_t>(units, (int64_t)num_sms() * std::max(per_sm, 1));
  kern<<<(unsigned)grid, RT, smem, st>>>(map, K, N, s, sw, Wq, error_word_ptr());
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  sqk::fold_scales_kernel<F8><<<(unsigned)((N + 255) / 256), 256, 0, st>>>(sw, N);
  return cudaGetLastError();
}

// Route of a fold: the one-shot cluster fold for bf16 W of at most 96 MiB whose cluster
// block fits; the streaming fold for other 16-byte-aligned bf16 W; the strip kernel
// otherwise.  Measured on W 4096 x {4096, 6144, 28672} and 14336 x 4096: the cluster fold
// leads below ~100 MB of W (23 against 25 us at 4096 x 4096), the streaming fold above
// (111 against 124 us at 4096 x 28672, 60 against 75 us at 14336 x 4096).
enum FoldRoute { FOLD_CLUSTER, FOLD_STREAM, FOLD_STRIPS };

static FoldRoute fold_route(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw, int* cw, int* cl, int* rk) {
  const bool tma_ok = bf16 && (reinterpret_cast<uintptr_t>(W) % 16) == 0 && (ldw * 2) % 16 == 0;
  if (!tma_ok) return FOLD_STRIPS;
  if (K * N * 2 <= (96ll << 20) && fold_cluster_shape(K, 72 * 1024, cw, cl, rk)) return FOLD_CLUSTER;
  return FOLD_STREAM;
}

int fold_kernel_launches(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw) {
  if (K <= 0 || N <= 0) return 0;
  int cw = 0, cl = 0, rk = 0;
  return fold_route(W, bf16, K, N, ldw, &cw, &cl, &rk) == FOLD_STREAM ? 3 : 1;
}

template <bool F8>
static cudaError_t launch_fold_any(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw, const float* s,
                                   const float* gamma, const float* beta, int8_t* Wq, float* sw, float* gamma_f,
                                   float* beta_f, cudaStream_t st) {
  int cw = 0, cl = 0, rk = 0;
  switch (fold_route(W, bf16, K, N, ldw, &cw, &cl, &rk)) {
    case FOLD_CLUSTER:
      switch (cw) {
        case 64: return launch_fold_cluster_t<64, F8>(W, K, N, ldw, cl, rk, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
        case 32: return launch_fold_cluster_t<32, F8>(W, K, N, ldw, cl, rk, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
        default: return launch_fold_cluster_t<16, F8>(W, K, N, ldw, cl, rk, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
      }
    case FOLD_STREAM:
      // 128-row tiles, one stage: seven 4-warp blocks per SM measured faster than deeper
      // rings with fewer blocks (111 against 125 us for 256-row tiles in a 2-stage ring)
      return launch_fold_stream<128, 1, F8>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
    default: break;
  }
  // narrower strips when there are few output channels, so every SM gets work
  const int64_t sms = num_sms();
  const int strip = (N / 32 >= 2 * sms) ? 32 : 16;
  if (bf16)
    return strip == 32 ? launch_fold_t<true, 32, F8>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st)
                       : launch_fold_t<true, 16, F8>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
  return strip == 32 ? launch_fold_t<false, 32, F8>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st)
                     : launch_fold_t<false, 16, F8>(W, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
}

cudaError_t launch_fold_quant(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw, const float* s,
                              const float* gamma, const float* beta, int8_t* Wq, float* sw, float* gamma_f,
                              float* beta_f, cudaStream_t st) {
  return launch_fold_any<false>(W, bf16, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, st);
}

// FP8 variant: E4M3 codes, sw = column max / 448.
cudaError_t launch_fold_quant_fp8(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw, const float* s,
                                  const float* gamma, const float* beta, uint8_t* Wq, float* sw, float* gamma_f,
                                  float* beta_f, cudaStream_t st) {
  return launch_fold_any<true>(W, bf16, K, N, ldw, s, gamma, beta, reinterpret_cast<int8_t*>(Wq), sw, gamma_f,
                               beta_f, st);
}

}  // namespace sqh

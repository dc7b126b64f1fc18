// sq_rowpipe.cu -- activation-row kernels with TMA bulk-copy staging:
//   LN_QUANT     fused LayerNorm (folded gamma' = gamma/s, beta' = beta/s) -> per-token INT8
//   PLAIN_QUANT  y = x / s (input from a previous GEMM)                     -> per-token INT8
//   LN_CALIB     per-channel absmax of LayerNorm(x) with the original gamma, beta
// ("4.2 W8A8 量化与 SmoothQuant", sec. 6 and 7.1; "量化：只压权重，与训练后量化（PTQ）",
// per-token activation quantisation.)
//
// A block of 256 threads holds 256 / T row groups of T threads.  Each group's first thread
// streams whole rows (cp.async.bulk, K * elt bytes) into the group's S-slot ring in shared
// memory, S rows ahead, completing on one mbarrier per slot; the per-channel vectors
// (gamma', beta' -- or s and RN(1/s) -- or gamma, beta) are copied to shared memory once per
// block.  A slot is refilled as soon as every thread of the group has moved its row into
// registers, which the row's first group barrier guarantees.  Row statistics use the fixed
// reduction order of sq_rowln.cuh; codes use the shared-divisor quantiser of sq_common.cuh.
#include <algorithm>

#include "sq_ptx.cuh"
#include "sq_rowln.cuh"

namespace sqk {

enum RowMode : int { ROW_LN_QUANT = 0, ROW_PLAIN_QUANT = 1, ROW_LN_CALIB = 2 };

template <bool BF16, int T, int NCH, int S, int MODE>
__global__ void __launch_bounds__(256)
rowpipe_kernel(const char* __restrict__ x, int64_t M, int K, int64_t ld_bytes, const float* __restrict__ vec_a,
               const float* __restrict__ vec_b, float eps, int8_t* __restrict__ xq, float* __restrict__ sx,
               float* __restrict__ out, const float* __restrict__ scale_in, int write_codes, unsigned int* err) {
  allow_dependent_launch();
  constexpr int G = 256 / T;
  constexpr int ELT = BF16 ? 2 : 4;
  constexpr bool LN = MODE != ROW_PLAIN_QUANT;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  float* sa = reinterpret_cast<float*>(sm);  // gamma' | s | gamma      [K]
  float* sb = sa + K;                          // beta'  | 1/s | beta     [K]
  const int row_bytes = K * ELT;
  uint8_t* ring = reinterpret_cast<uint8_t*>(sb + K);  // [G][S][row_bytes]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ring + (size_t)G * S * row_bytes);  // [G][S]
  __shared__ float red[G][24];
  __shared__ int stop[G];  // a group's wait ran out: it takes no further rows

  const int gid = threadIdx.x / T, t = threadIdx.x % T;
  const int nchunks = K / 8;
  const unsigned long long limit = wait_limit(err);
  if (t == 0) stop[gid] = 0;

  // per-channel vectors, once per block, as float4s ordered [half][chunk] (element j sits at
  // ((j % 8) / 4 * nchunks + j / 8) * 4 + j % 4) so that a thread's read of its chunk's half
  // h is 16 bytes after its neighbour's: conflict-free.
  int slow = 0;
  for (int j = threadIdx.x; j < K; j += 256) {
    const int at = (((j & 7) >> 2) * nchunks + (j >> 3)) * 4 + (j & 3);
    const float a = vec_a[j];
    sa[at] = a;
    if (MODE == ROW_PLAIN_QUANT) {
      const bool fast = fabsf(a) >= 0x1p-90f && fabsf(a) <= 0x1p+90f;
      slow |= !fast;
      sb[at] = fast ? __frcp_rn(a) : 0.0f;
    } else {
      sb[at] = vec_b ? vec_b[j] : 0.0f;
    }
  }
  if (t == 0) {
    for (int k = 0; k < S; ++k) mbar_init(smem_u32(&bars[gid * S + k]), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  const bool all_fast = !__syncthreads_or(slow);

  uint8_t* gring = ring + (size_t)gid * S * row_bytes;
  const int64_t rstep = (int64_t)gridDim.x * G;
  const int64_t r0 = (int64_t)blockIdx.x * G + gid;
  auto issue = [&](int slot, int64_t r) {
    const uint32_t b = smem_u32(&bars[gid * S + slot]);
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    mbar_arrive_expect_tx(b, (uint32_t)row_bytes);
    bulk_load(smem_u32(gring + (size_t)slot * row_bytes), x + r * ld_bytes, (uint32_t)row_bytes, b);
  };
  if (t == 0)
    for (int k = 0; k < S; ++k)
      if (r0 + k * rstep < M) issue(k, r0 + k * rstep);

  float cm[MODE == ROW_LN_CALIB ? NCH * 8 : 1];
  if (MODE == ROW_LN_CALIB) {
#pragma unroll
    for (int i = 0; i < NCH * 8; ++i) cm[i] = 0.0f;
  }

  int64_t it = 0;
  for (int64_t r = r0; r < M; r += rstep, ++it) {
    const int slot = (int)(it % S);
    // one lane polls the slot's barrier; the rest of the group sleeps in the group barrier
    if (t == 0 && !mbar_wait(smem_u32(&bars[gid * S + slot]), (uint32_t)((it / S) & 1), limit)) {
      atomicOr(err, ERR_ROW_TMA_WAIT);
      stop[gid] = 1;
    }
    group_barrier<T>(gid);
    if (stop[gid]) {
      // the group stops: the copies it has issued (rows it .. it + S - 1) land before it leaves
      if (t == 0)
        for (int j = 0; j < S; ++j)
          if (r + j * rstep < M)
            (void)mbar_wait(smem_u32(&bars[gid * S + (int)((it + j) % S)]), (uint32_t)(((it + j) / S) & 1), DRAIN_NS);
      group_barrier<T>(gid);
      break;
    }
    const uint8_t* rowp = gring + (size_t)slot * row_bytes;
    float v[NCH * 8];
#pragma unroll
    for (int m = 0; m < NCH; ++m) {
      const int c = t + T * m;
      if (c < nchunks) {
        if (BF16) {
          unpack8_bf16(*reinterpret_cast<const uint4*>(rowp + (size_t)c * 16), v + m * 8);
        } else {
          const uint4 a = *reinterpret_cast<const uint4*>(rowp + (size_t)c * 32);
          const uint4 b = *reinterpret_cast<const uint4*>(rowp + (size_t)c * 32 + 16);
          v[m * 8 + 0] = __uint_as_float(a.x); v[m * 8 + 1] = __uint_as_float(a.y);
          v[m * 8 + 2] = __uint_as_float(a.z); v[m * 8 + 3] = __uint_as_float(a.w);
          v[m * 8 + 4] = __uint_as_float(b.x); v[m * 8 + 5] = __uint_as_float(b.y);
          v[m * 8 + 6] = __uint_as_float(b.z); v[m * 8 + 7] = __uint_as_float(b.w);
        }
      }
    }
    // ---- y in v[]
    if (LN) {
      float rstd;
      group_row_stats_d<T, NCH>(v, nchunks, K, eps, red[gid], t, gid, rstd);  // v <- x - mu
      if (t == 0 && r + S * rstep < M) issue(slot, r + S * rstep);           // slot drained
#pragma unroll
      for (int m = 0; m < NCH; ++m) {
        const int c = t + T * m;
        if (c < nchunks) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float4 g = *reinterpret_cast<const float4*>(sa + (h * nchunks + c) * 4);
            const float4 b = *reinterpret_cast<const float4*>(sb + (h * nchunks + c) * 4);
            float* d = v + m * 8 + h * 4;
            const float2 rs2 = make_float2(rstd, rstd);
            const float2 y01 = __ffma2_rn(__fmul2_rn(make_float2(d[0], d[1]), rs2), make_float2(g.x, g.y),
                                          make_float2(b.x, b.y));
            const float2 y23 = __ffma2_rn(__fmul2_rn(make_float2(d[2], d[3]), rs2), make_float2(g.z, g.w),
                                          make_float2(b.z, b.w));
            d[0] = y01.x; d[1] = y01.y; d[2] = y23.x; d[3] = y23.y;
          }
        }
      }
    } else {
#pragma unroll
      for (int m = 0; m < NCH; ++m) {
        const int c = t + T * m;
        if (c < nchunks) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float4 sv = *reinterpret_cast<const float4*>(sa + (h * nchunks + c) * 4);
            const float4 rv = *reinterpret_cast<const float4*>(sb + (h * nchunks + c) * 4);
            float* d = v + m * 8 + h * 4;
            if (all_fast) {
              // Markstein: q = RN(x y), r = x - s q exact, RN(q + r y) = RN(x / s), two lanes at a time
              const float2 x01 = make_float2(d[0], d[1]), x23 = make_float2(d[2], d[3]);
              const float2 r01 = make_float2(rv.x, rv.y), r23 = make_float2(rv.z, rv.w);
              const float2 y01 = markstein2(x01, r01, make_float2(-sv.x, -sv.y));
              const float2 y23 = markstein2(x23, r23, make_float2(-sv.z, -sv.w));
              d[0] = y01.x; d[1] = y01.y; d[2] = y23.x; d[3] = y23.y;
            } else {
              d[0] = __fdiv_rn(d[0], sv.x);
              d[1] = __fdiv_rn(d[1], sv.y);
              d[2] = __fdiv_rn(d[2], sv.z);
              d[3] = __fdiv_rn(d[3], sv.w);
            }
          }
        }
      }
    }
    if (MODE == ROW_LN_CALIB) {
#pragma unroll
      for (int m = 0; m < NCH; ++m)
        if (t + T * m < nchunks)
#pragma unroll
          for (int e = 0; e < 8; ++e) cm[m * 8 + e] = fmaxf(cm[m * 8 + e], fabsf(v[m * 8 + e]));
      continue;
    }
    // ---- per-token quantisation
    float am[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 8 independent max chains
#pragma unroll
    for (int m = 0; m < NCH; ++m)
      if (t + T * m < nchunks)
#pragma unroll
        for (int e = 0; e < 8; ++e) am[e] = fmaxf(am[e], fabsf(v[m * 8 + e]));
    float amax = fmaxf(fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3])), fmaxf(fmaxf(am[4], am[5]), fmaxf(am[6], am[7])));
    amax = group_max<T>(amax, red[gid] + 16, t, gid);
    if (!LN && t == 0 && r + S * rstep < M) issue(slot, r + S * rstep);  // slot drained
    // per-token scale, or the per-tensor scale handed in (then codes clamp at +-127)
    const float scale = scale_in ? __ldg(scale_in) : __fdiv_rn(amax, 127.0f);
    if (t == 0) sx[r] = scale;
    if (write_codes) store_row_codes<T, NCH>(v, t, nchunks, scale, scale_in != nullptr, xq + r * (int64_t)K);
  }

  if (MODE == ROW_LN_CALIB) {
    // merge the groups' column maxima through shared memory (the ring is idle now), then
    // one atomicMax per column per block
    __syncthreads();
    float* scratch = reinterpret_cast<float*>(ring);  // [G][K]
#pragma unroll
    for (int m = 0; m < NCH; ++m) {
      const int c = t + T * m;
      if (c < nchunks)
#pragma unroll
        for (int e = 0; e < 8; ++e) scratch[gid * K + c * 8 + e] = cm[m * 8 + e];
    }
    __syncthreads();
    if ((int64_t)blockIdx.x * G < M)
      for (int j = threadIdx.x; j < K; j += 256) {
        float mx = scratch[j];
#pragma unroll
        for (int g = 1; g < G; ++g) mx = fmaxf(mx, scratch[g * K + j]);
        atomic_max_nonneg(out + j, mx);
      }
  }
}

}  // namespace sqk

namespace sqh {

int pick_row_threads(int64_t K, int max_nch, int* nch);

// Shared memory of one block: two per-channel vectors, the rings, the barriers.
static size_t rowpipe_smem(int K, int elt, int G, int S) {
  return 128 + (size_t)K * 8 + (size_t)G * S * K * elt + (size_t)G * S * 8;
}

template <bool BF16, int T, int NCH, int MODE, int S>
static cudaError_t launch_rowpipe_v(const void* x, int64_t M, int K, int64_t ld_bytes, const float* va,
                                    const float* vb, float eps, int8_t* xq, float* sx, float* out, const float* scale_in,
                                    int write_codes, cudaStream_t st) {
  constexpr int G = 256 / T;
  auto kern = sqk::rowpipe_kernel<BF16, T, NCH, S, MODE>;
  const size_t smem = rowpipe_smem(K, BF16 ? 2 : 4, G, S);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (M + G - 1) / G;
  const int64_t grid = std::min<int64_t>(blocks, (int64_t)num_sms() * std::max(per_sm, 1));
  kern<<<(unsigned)grid, 256, smem, st>>>((const char*)x, M, K, ld_bytes, va, vb, eps, xq, sx, out, scale_in,
                                          write_codes, error_word_ptr());
  return cudaGetLastError();
}

// Two ring slots per group; one lane per group polls the slot barrier while the rest of the
// group waits in the hardware group barrier (measured best of {2, 3} slots x {one, all} pollers).
template <bool BF16, int T, int NCH, int MODE>
static cudaError_t launch_rowpipe_t(const void* x, int64_t M, int K, int64_t ld_bytes, const float* va,
                                    const float* vb, float eps, int8_t* xq, float* sx, float* out,
                                    const float* scale_in, int write_codes, cudaStream_t st) {
  return launch_rowpipe_v<BF16, T, NCH, MODE, 2>(x, M, K, ld_bytes, va, vb, eps, xq, sx, out, scale_in,
                                                 write_codes, st);
}

template <bool BF16, int T, int MODE>
static cudaError_t launch_rowpipe_nch(int nch, const void* x, int64_t M, int K, int64_t ld_bytes, const float* va,
                                      const float* vb, float eps, int8_t* xq, float* sx, float* out,
                                      const float* scale_in, int write_codes, cudaStream_t st) {
#define SQ_RP(N) launch_rowpipe_t<BF16, T, N, MODE>(x, M, K, ld_bytes, va, vb, eps, xq, sx, out, scale_in, write_codes, st)
  if (nch <= 1) return SQ_RP(1);
  if (nch <= 2) return SQ_RP(2);
  if (nch <= 4) return SQ_RP(4);
  // calibration keeps at most 4 chunks per thread (its running maxima live in registers too)
  if (MODE == sqk::ROW_LN_CALIB) return cudaErrorInvalidValue;
  constexpr int N8 = MODE == sqk::ROW_LN_CALIB ? 4 : 8;
  return SQ_RP(N8);
#undef SQ_RP
}

template <int MODE>
static cudaError_t launch_rowpipe_mode(bool bf16, int T, int nch, const void* x, int64_t M, int K, int64_t ld_bytes,
                                       const float* va, const float* vb, float eps, int8_t* xq, float* sx, float* out,
                                       const float* scale_in, int write_codes, cudaStream_t st) {
#define SQ_T(TT)                                                                                                 \
  if (T == TT)                                                                                                   \
    return bf16 ? launch_rowpipe_nch<true, TT, MODE>(nch, x, M, K, ld_bytes, va, vb, eps, xq, sx, out, scale_in,  \
                                                    write_codes, st)                                             \
                : launch_rowpipe_nch<false, TT, MODE>(nch, x, M, K, ld_bytes, va, vb, eps, xq, sx, out, scale_in, \
                                                     write_codes, st);
  SQ_T(32) SQ_T(64) SQ_T(128) SQ_T(256)
#undef SQ_T
  return cudaErrorInvalidValue;
}

// Whether the staged row kernel applies (rows of up to 8 chunks per thread whose block fits
// the shared memory); sets threads per row and chunks per thread.
bool rowpipe_shape(int64_t K, bool bf16, int max_nch, int* T, int* nch) {
  *T = pick_row_threads(K, max_nch, nch);
  if (!*T) return false;
  return rowpipe_smem((int)K, bf16 ? 2 : 4, 256 / *T, 2) <= 200 * 1024;
}

cudaError_t launch_rowpipe_quant(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                                 const float* beta_f, const float* s, float eps, int8_t* xq, float* sx, int T, int nch,
                                 const float* scale_in, int write_codes, cudaStream_t st) {
  const int64_t ldb = ldx * (bf16 ? 2 : 4);
  if (gamma_f)
    return launch_rowpipe_mode<sqk::ROW_LN_QUANT>(bf16, T, nch, x, M, (int)K, ldb, gamma_f, beta_f, eps, xq, sx,
                                                  nullptr, scale_in, write_codes, st);
  return launch_rowpipe_mode<sqk::ROW_PLAIN_QUANT>(bf16, T, nch, x, M, (int)K, ldb, s, nullptr, eps, xq, sx, nullptr,
                                                   scale_in, write_codes, st);
}

cudaError_t launch_rowpipe_calib(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ldx, const float* gamma,
                                 const float* beta, float eps, float* out, int T, int nch, cudaStream_t st) {
  const int64_t ldb = ldx * (bf16 ? 2 : 4);
  return launch_rowpipe_mode<sqk::ROW_LN_CALIB>(bf16, T, nch, x, rows, (int)K, ldb, gamma, beta, eps, nullptr, nullptr,
                                                out, nullptr, 1, st);
}

}  // namespace sqh

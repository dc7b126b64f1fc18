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

// Blocks loop over rows (grid sized to the resident blocks); with PREFETCH the next row's
// loads are issued before the current row is reduced, so HBM stays busy during the
// block-wide reductions.  With KEEP_Y the row's y values stay in registers between the
// absmax and the quantisation (computed once); otherwise they are recomputed.
// F8: E4M3 codes with scale = max / 448 (the FP8 variant) instead of INT8 with max / 127.
template <bool BF16, int MAXC, bool LN, bool PREFETCH, bool KEEP_Y, bool F8 = false>
__global__ void __launch_bounds__(ROW_THREADS)
ln_smooth_quant_kernel(const char* __restrict__ x, int64_t M, int K, int64_t ld_bytes,
                       const float* __restrict__ gamma_f, const float* __restrict__ beta_f,
                       const float* __restrict__ s, float eps, int8_t* __restrict__ xq, float* __restrict__ sx,
                       const float* __restrict__ scale_in, int write_codes) {
  allow_dependent_launch();
  __shared__ float red[3 * (ROW_WARPS + 1)];
  const int nchunks = K / 8;
  RowChunks<BF16, MAXC> cur;
  int64_t m = blockIdx.x;
  if (m < M) cur.load(x + m * ld_bytes, nchunks);
  for (; m < M; m += gridDim.x) {
    const int64_t mn = m + gridDim.x;
    RowChunks<BF16, MAXC> nxt;
    if (PREFETCH && mn < M) nxt.load(x + mn * ld_bytes, nchunks);
    float mu = 0.0f, rstd = 0.0f;
    if (LN) row_stats(cur, nchunks, K, eps, red, mu, rstd);
    float yk[KEEP_Y ? MAXC * 8 : 1];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = threadIdx.x + i * ROW_THREADS;
      if (c < nchunks) {
        float f[8], y[8];
        cur.get(i, f);
        if (LN) ln_chunk(f, mu, rstd, gamma_f, beta_f, c, y);
        else div_chunk(f, s, c, y);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          amax = fmaxf(amax, fabsf(y[e]));
          if (KEEP_Y) yk[i * 8 + e] = y[e];
        }
      }
    }
    amax = block_max(amax, red + 2 * (ROW_WARPS + 1));
    const float scale = scale_in ? __ldg(scale_in) : __fdiv_rn(amax, F8 ? 448.0f : 127.0f);
    const SharedDivisor d(scale);
    if (threadIdx.x == 0) sx[m] = scale;
    int8_t* qrow = xq + m * (int64_t)K;
#pragma unroll
    for (int i = 0; i < (write_codes ? MAXC : 0); ++i) {
      const int c = threadIdx.x + i * ROW_THREADS;
      if (c < nchunks) {
        float y[8];
        if (KEEP_Y) {
#pragma unroll
          for (int e = 0; e < 8; ++e) y[e] = yk[i * 8 + e];
        } else {
          float f[8];
          cur.get(i, f);
          if (LN) ln_chunk(f, mu, rstd, gamma_f, beta_f, c, y);
          else div_chunk(f, s, c, y);
        }
        if (F8)
          *reinterpret_cast<uint2*>(qrow + (int64_t)c * 8) = d.fast ? pack8_e4m3<true>(y, d) : pack8_e4m3<false>(y, d);
        else
          *reinterpret_cast<uint2*>(qrow + (int64_t)c * 8) = pack8_codes<false, true>(y, d);
      }
    }
    if (PREFETCH) cur = nxt;
    else if (mn < M) cur.load(x + mn * ld_bytes, nchunks);
  }
}

// Rows of up to 16384 elements: one group of T threads per row (256 / T rows per block),
// the row as floats in registers, the next row's raw vectors loaded as soon as the
// current row is converted; y overwrites x in place.
template <bool BF16, int T, int NCH, bool LN>
__global__ void __launch_bounds__(256, 2)
ln_quant_group_kernel(const char* __restrict__ x, int64_t M, int K, int64_t ld_bytes,
                      const float* __restrict__ gamma_f, const float* __restrict__ beta_f,
                      const float* __restrict__ s, float eps, int8_t* __restrict__ xq, float* __restrict__ sx,
                      const float* __restrict__ scale_in, int write_codes, int use_table) {
  allow_dependent_launch();
  constexpr int G = 256 / T;
  __shared__ float red[G][24];  // per group: mean partials, variance partials, max
  extern __shared__ float rs[];  // plain mode: RN(1 / s_j), or 0 where s_j is outside the fast range
  const int gid = threadIdx.x / T, t = threadIdx.x % T;
  const int nchunks = K / 8;
  // plain mode: a table of RN(1/s_j) pays off over several rows per block; with a row or two
  // (decode) the correctly rounded division per element is cheaper than building it
  bool all_fast = LN || use_table;
  if (!LN && use_table) {
    int slow = 0;
    for (int j = threadIdx.x; j < K; j += 256) {
      const float a = s[j];
      const bool fast = fabsf(a) >= 0x1p-90f && fabsf(a) <= 0x1p+90f;
      slow |= !fast;
      rs[(((j & 7) >> 2) * nchunks + (j >> 3)) * 4 + (j & 3)] = fast ? __frcp_rn(a) : 0.0f;  // [half][chunk]
    }
    all_fast = !__syncthreads_or(slow);
  }
  RowRaw<BF16, NCH> raw;
  const int64_t mstep = (int64_t)gridDim.x * G;
  int64_t m = (int64_t)blockIdx.x * G + gid;
  if (m < M) raw.template load<T>(x + m * ld_bytes, nchunks, t);
  for (; m < M; m += mstep) {
    float v[NCH * 8];
    raw.to_float(v);
    const int64_t mn = m + mstep;
    if (mn < M) raw.template load<T>(x + mn * ld_bytes, nchunks, t);
    float mu = 0.0f, rstd = 0.0f;
    if (LN) group_row_stats<T, NCH>(v, nchunks, K, eps, red[gid], t, gid, mu, rstd);
    float am[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};  // 8 independent max chains
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = t + T * i;
      if (c < nchunks) {
        if (LN) {
          ln_chunk(v + i * 8, mu, rstd, gamma_f, beta_f, c, v + i * 8);
        } else if (all_fast) {
          // y = x / s_j through the shared divisor s_j with y_j = RN(1/s_j) (Markstein)
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const float4 sv = __ldg(reinterpret_cast<const float4*>(s + (size_t)c * 8 + h * 4));
            const float4 rv = *reinterpret_cast<const float4*>(rs + (h * nchunks + c) * 4);
            float* d = v + i * 8 + h * 4;
            float q;
            q = __fmul_rn(d[0], rv.x); d[0] = __fmaf_rn(__fmaf_rn(-q, sv.x, d[0]), rv.x, q);
            q = __fmul_rn(d[1], rv.y); d[1] = __fmaf_rn(__fmaf_rn(-q, sv.y, d[1]), rv.y, q);
            q = __fmul_rn(d[2], rv.z); d[2] = __fmaf_rn(__fmaf_rn(-q, sv.z, d[2]), rv.z, q);
            q = __fmul_rn(d[3], rv.w); d[3] = __fmaf_rn(__fmaf_rn(-q, sv.w, d[3]), rv.w, q);
          }
        } else {
          div_chunk(v + i * 8, s, c, v + i * 8);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) am[e] = fmaxf(am[e], fabsf(v[i * 8 + e]));
      }
    }
    float amax = fmaxf(fmaxf(fmaxf(am[0], am[1]), fmaxf(am[2], am[3])), fmaxf(fmaxf(am[4], am[5]), fmaxf(am[6], am[7])));
    amax = group_max<T>(amax, red[gid] + 16, t, gid);
    const float scale = scale_in ? __ldg(scale_in) : __fdiv_rn(amax, 127.0f);
    if (t == 0) sx[m] = scale;
    if (write_codes) store_row_codes<T, NCH>(v, t, nchunks, scale, scale_in != nullptr, xq + m * (int64_t)K);
  }
}


// ---------------------------------------------------------------------------- long plain rows
// Plain mode (y = x / s) on rows too long to hold in a thread group's registers (K > 16384).
// A block owns one segment of SEG_CH channels and strides over the rows (row p, p + P, ...).
// Each thread keeps s and RN(1/s) of its SEG_CH / 2048 chunks in registers for all its rows,
// so that y = RN(x / s) takes Markstein's three operations per element instead of a full
// division (divisors outside the fast range fall back to the division, for the whole block).
// Pass 1 folds each (row, segment) maximum of |y| into the row's slot of sx (float bits,
// atomicMax; sx starts at 0); pass 2 recomputes y and writes the codes with scale =
// RN(max / 127) (or the given per-tensor scale, codes clamped); pass 3 turns the maxima in sx
// into scales.  Two rows per step, the next two rows' loads in flight behind them.
// (One block per (row, segment) with a division per element: 153 us at 2048 x 49152.)
constexpr int SEG_CH = 4096;                   // channels per segment
constexpr int SEG_CPT = SEG_CH / 8 / 256;      // chunks per thread
constexpr int SEG_CHUNKS = SEG_CH / 8;

template <bool BF16>
__device__ __forceinline__ void seg_load_raw(const char* row, int64_t c, uint4* v) {
  if (BF16) {
    v[0] = ldg_stream16(row + c * 16);
  } else {
    v[0] = ldg_stream16(row + c * 32);
    v[1] = ldg_stream16(row + c * 32 + 16);
  }
}

template <bool BF16>
__device__ __forceinline__ void seg_unpack(const uint4* v, float f[8]) {
  if (BF16) {
    unpack8_bf16(v[0], f);
  } else {
    f[0] = __uint_as_float(v[0].x); f[1] = __uint_as_float(v[0].y);
    f[2] = __uint_as_float(v[0].z); f[3] = __uint_as_float(v[0].w);
    f[4] = __uint_as_float(v[1].x); f[5] = __uint_as_float(v[1].y);
    f[6] = __uint_as_float(v[1].z); f[7] = __uint_as_float(v[1].w);
  }
}

// Per-thread channel constants of a segment: chunks c = seg * SEG_CHUNKS + t + 256 i.
struct SegConst {
  float s[SEG_CPT][8], rc[SEG_CPT][8];
  bool ok[SEG_CPT];
};

__device__ __forceinline__ bool seg_const(SegConst& sc, const float* __restrict__ s, int64_t seg, int64_t nchunks) {
  bool slow = false;
#pragma unroll
  for (int i = 0; i < SEG_CPT; ++i) {
    const int64_t c = seg * SEG_CHUNKS + threadIdx.x + 256 * i;
    sc.ok[i] = c < nchunks;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float a = sc.ok[i] ? __ldg(s + c * 8 + e) : 1.0f;
      const bool fast = fabsf(a) >= 0x1p-90f && fabsf(a) <= 0x1p+90f;
      slow |= !fast;
      sc.s[i][e] = a;
      sc.rc[i][e] = fast ? __frcp_rn(a) : 0.0f;
    }
  }
  return slow;
}

// y = RN(x / s) for chunk i of the thread (FAST: Markstein on packed pairs).  SIGNED: the E4M3
// codes tell -0 from +0, and RN(-0 / s) = -0, which Markstein's correction turns into +0.
template <bool FAST, bool SIGNED>
__device__ __forceinline__ void seg_div(const SegConst& sc, int i, const float f[8], float y[8]) {
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    if (FAST) {
      const float2 q = markstein2(make_float2(f[e], f[e + 1]), make_float2(sc.rc[i][e], sc.rc[i][e + 1]),
                                  make_float2(-sc.s[i][e], -sc.s[i][e + 1]));
      y[e] = SIGNED ? with_sign_of(q.x, f[e]) : q.x;
      y[e + 1] = SIGNED ? with_sign_of(q.y, f[e + 1]) : q.y;
    } else {
      y[e] = __fdiv_rn(f[e], sc.s[i][e]);
      y[e + 1] = __fdiv_rn(f[e + 1], sc.s[i][e + 1]);
    }
  }
}

template <bool BF16>
__device__ __forceinline__ void seg_load_rows(const char* x, int64_t ld_bytes, int64_t r, int64_t M, int64_t seg,
                                              const SegConst& sc, uint4 (&v)[2][SEG_CPT][BF16 ? 1 : 2]) {
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int i = 0; i < SEG_CPT; ++i)
      if (r + h < M && sc.ok[i])
        seg_load_raw<BF16>(x + (r + h) * ld_bytes, seg * SEG_CHUNKS + threadIdx.x + 256 * i, v[h][i]);
}

// PASS 0: row maxima into rowmax; PASS 1: codes.  Block b: segment b % nseg, rows b / nseg,
// b / nseg + P, ... in pairs (P = gridDim.x / nseg).
template <bool BF16, int PASS, bool F8>
__global__ void __launch_bounds__(256)
rowsplit_kernel(const char* __restrict__ x, int64_t M, int64_t K, int64_t ld_bytes, int64_t nseg,
                const float* __restrict__ s, float* __restrict__ rowmax, const float* __restrict__ scale_in,
                int8_t* __restrict__ xq) {
  allow_dependent_launch();
  constexpr int V = BF16 ? 1 : 2;
  __shared__ float red[2][2][8];  // [step parity][row of the pair][warp]
  const int64_t seg = blockIdx.x % nseg, p = blockIdx.x / nseg, P = gridDim.x / nseg;
  const int64_t nchunks = K / 8;
  SegConst sc;
  const bool fast = !__syncthreads_or(seg_const(sc, s, seg, nchunks));
  uint4 v[2][SEG_CPT][V], nv[2][SEG_CPT][V];
  int64_t r = 2 * p;
  if (r < M) seg_load_rows<BF16>(x, ld_bytes, r, M, seg, sc, v);
  for (int step = 0; r < M; r += 2 * P, ++step) {
    const int64_t rn = r + 2 * P;
    if (rn < M) seg_load_rows<BF16>(x, ld_bytes, rn, M, seg, sc, nv);
    if constexpr (PASS == 0) {
      float am[2] = {0.0f, 0.0f};
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int i = 0; i < SEG_CPT; ++i)
          if (r + h < M && sc.ok[i]) {
            float f[8], y[8];
            seg_unpack<BF16>(v[h][i], f);
            if (fast) seg_div<true, false>(sc, i, f, y);
            else seg_div<false, false>(sc, i, f, y);
#pragma unroll
            for (int e = 0; e < 8; ++e) am[h] = fmaxf(am[h], fabsf(y[e]));
          }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) am[h] = fmaxf(am[h], __shfl_xor_sync(0xffffffffu, am[h], o));
        if ((threadIdx.x & 31) == 0) red[step & 1][h][threadIdx.x >> 5] = am[h];
      }
      __syncthreads();  // red[step & 1] is rewritten two steps later, after the next barrier
      if (threadIdx.x < 2 && r + threadIdx.x < M) {
        float m = red[step & 1][threadIdx.x][0];
#pragma unroll
        for (int w = 1; w < 8; ++w) m = fmaxf(m, red[step & 1][threadIdx.x][w]);
        atomic_max_nonneg(rowmax + r + threadIdx.x, m);
      }
    } else {
      const bool clamp = scale_in != nullptr;
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        if (r + h >= M) continue;
        const float scale = clamp ? __ldg(scale_in) : __fdiv_rn(__ldg(rowmax + r + h), F8 ? 448.0f : 127.0f);
        const SharedDivisor d(scale);
        int8_t* qrow = xq + (r + h) * K;
#pragma unroll
        for (int i = 0; i < SEG_CPT; ++i) {
          if (!sc.ok[i]) continue;
          float f[8], y[8];
          seg_unpack<BF16>(v[h][i], f);
          if (fast) seg_div<true, F8>(sc, i, f, y);
          else seg_div<false, F8>(sc, i, f, y);
          uint2 w;
          if (F8) w = d.fast ? pack8_e4m3<true>(y, d) : pack8_e4m3<false>(y, d);
          else if (d.fast && !clamp) w = pack8_codes<true>(y, d);
          else if (d.fast) w = pack8_codes<true, true>(y, d);
          else w = pack8_codes<false, true>(y, d);
          *reinterpret_cast<uint2*>(qrow + (seg * SEG_CHUNKS + threadIdx.x + 256 * i) * 8) = w;
        }
      }
    }
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int i = 0; i < SEG_CPT; ++i)
#pragma unroll
        for (int u = 0; u < V; ++u) v[h][i][u] = nv[h][i][u];
  }
}

// sx[m] = RN(max_m / 127) (F8: / 448), or the given per-tensor scale.
template <bool F8>
__global__ void rowsplit_scales_kernel(float* __restrict__ sx, int64_t M, const float* __restrict__ scale_in) {
  allow_dependent_launch();
  const int64_t m = (int64_t)blockIdx.x * 256 + threadIdx.x;
  if (m < M) sx[m] = scale_in ? __ldg(scale_in) : __fdiv_rn(sx[m], F8 ? 448.0f : 127.0f);
}

// out[0] = max of v[0 .. n) (non-negative floats), one block.
__global__ void __launch_bounds__(1024) max_of_vector_kernel(const float* __restrict__ v, int64_t n, float* out) {
  allow_dependent_launch();
  __shared__ float red[32];
  float m = 0.0f;
  for (int64_t i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, v[i]);
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = red[threadIdx.x];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (threadIdx.x == 0) out[0] = m;
  }
}

}  // namespace sqk

namespace sqh {

template <bool BF16, int T, int NCH, bool LN>
static cudaError_t launch_group_t(const void* x, int64_t M, int K, int64_t ld_bytes, const float* gamma_f,
                                  const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                                  const float* scale_in, int write_codes, cudaStream_t st) {
  auto kern = sqk::ln_quant_group_kernel<BF16, T, NCH, LN>;
  const size_t table = LN ? 0 : sizeof(float) * (size_t)K;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)table);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, table);
  if (e != cudaSuccess) return e;
  constexpr int G = 256 / T;
  const int64_t blocks = (M + G - 1) / G;
  const int64_t grid = std::min<int64_t>(blocks, (int64_t)num_sms() * std::max(per_sm, 1));
  const int use_table = !LN && M >= 4 * grid * G;  // at least 4 rows per group
  kern<<<(unsigned)grid, 256, use_table ? table : 0, st>>>((const char*)x, M, K, ld_bytes, gamma_f, beta_f, s, eps,
                                                           xq, sx, scale_in, write_codes, use_table);
  return cudaGetLastError();
}

template <bool BF16, int T>
static cudaError_t launch_group_nch(int nch, const void* x, int64_t M, int K, int64_t ld_bytes, const float* gamma_f,
                                    const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                                    const float* scale_in, int write_codes, cudaStream_t st) {
#define SQ_GRP(NCH)                                                                                                \
  if (nch <= NCH)                                                                                                  \
    return gamma_f ? launch_group_t<BF16, T, NCH, true>(x, M, K, ld_bytes, gamma_f, beta_f, s, eps, xq, sx, scale_in, \
                                                        write_codes, st)                                           \
                   : launch_group_t<BF16, T, NCH, false>(x, M, K, ld_bytes, gamma_f, beta_f, s, eps, xq, sx, scale_in, \
                                                         write_codes, st);
  SQ_GRP(1) SQ_GRP(2) SQ_GRP(4) SQ_GRP(6) SQ_GRP(7) SQ_GRP(8)
#undef SQ_GRP
  return cudaErrorInvalidValue;
}

// Threads per row for the group kernels: the smallest T whose chunks per thread fit in
// `max_nch`; 0 when even T = 256 does not.
int pick_row_threads(int64_t K, int max_nch, int* nch) {
  const int64_t nchunks = K / 8;
  for (int T : {32, 64, 128, 256}) {
    const int64_t n = (nchunks + T - 1) / T;
    if (n <= max_nch) {
      *nch = (int)n;
      return T;
    }
  }
  return 0;
}

template <bool BF16, int MAXC, bool LN, bool F8 = false>
static cudaError_t launch_lnq_mode(const void* x, int64_t M, int K, int64_t ld_bytes, const float* gamma_f,
                                   const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                                   const float* scale_in, int write_codes, cudaStream_t st) {
  constexpr bool PF = BF16 && MAXC <= 4;      // register double buffer while it stays small
  constexpr bool KEEP = MAXC <= 8;            // y in registers (64 floats at most)
  auto kern = sqk::ln_smooth_quant_kernel<BF16, MAXC, LN, PF, KEEP, F8>;
  int per_sm = 1;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, sqk::ROW_THREADS, 0);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(M, (int64_t)num_sms() * std::max(per_sm, 1));
  kern<<<(unsigned)grid, sqk::ROW_THREADS, 0, st>>>((const char*)x, M, K, ld_bytes, gamma_f, beta_f, s, eps, xq,
                                                    sx, scale_in, write_codes);
  return cudaGetLastError();
}

template <bool BF16, int MAXC, bool F8 = false>
static cudaError_t launch_lnq_t(const void* x, int64_t M, int K, int64_t ld_bytes, const float* gamma_f,
                                const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                                const float* scale_in, int write_codes, cudaStream_t st) {
  if (gamma_f)
    return launch_lnq_mode<BF16, MAXC, true, F8>(x, M, K, ld_bytes, gamma_f, beta_f, s, eps, xq, sx, scale_in,
                                                 write_codes, st);
  return launch_lnq_mode<BF16, MAXC, false, F8>(x, M, K, ld_bytes, gamma_f, beta_f, s, eps, xq, sx, scale_in,
                                                write_codes, st);
}

bool rowpipe_shape(int64_t K, bool bf16, int max_nch, int* T, int* nch);
cudaError_t launch_rowpipe_quant(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                                 const float* beta_f, const float* s, float eps, int8_t* xq, float* sx, int T, int nch,
                                 const float* scale_in, int write_codes, cudaStream_t st);

bool rowpair_supported(int64_t K, bool bf16, bool calib, int64_t rows);
cudaError_t launch_rowpair_quant(const void* x, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                                 const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                                 const float* scale_in, int write_codes, bool f8, cudaStream_t st);


// Plain-mode rows longer than the register-resident kernels hold (see rowsplit_kernel).  F8:
// E4M3 codes, scale = max / 448.
template <bool F8>
static cudaError_t launch_rowsplit(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, const float* s,
                                   int8_t* xq, float* sx, const float* scale_in, int write_codes, cudaStream_t st) {
  const int64_t ldb = ldx * (bf16 ? 2 : 4);
  const int64_t nseg = (K / 8 + sqk::SEG_CHUNKS - 1) / sqk::SEG_CHUNKS;
  // one wave: the row pairs of a segment spread over as many blocks as are resident at once
  int per_sm = 1;
  cudaError_t e = bf16 ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sqk::rowsplit_kernel<true, 0, F8>, 256, 0)
                       : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, sqk::rowsplit_kernel<false, 0, F8>, 256, 0);
  if (e != cudaSuccess) return e;
  const int64_t pairs = (M + 1) / 2;
  const int64_t per_seg = std::max<int64_t>(1, std::min<int64_t>(pairs, (int64_t)num_sms() * std::max(per_sm, 1) / nseg));
  const int64_t blocks = nseg * per_seg;
  if (blocks > INT32_MAX) return cudaErrorInvalidValue;
  const char* xb = (const char*)x;
  if (!scale_in) {  // per-token maxima into sx
    e = cudaMemsetAsync(sx, 0, sizeof(float) * (size_t)M, st);
    if (e != cudaSuccess) return e;
    if (bf16) sqk::rowsplit_kernel<true, 0, F8><<<(unsigned)blocks, 256, 0, st>>>(xb, M, K, ldb, nseg, s, sx, scale_in, xq);
    else sqk::rowsplit_kernel<false, 0, F8><<<(unsigned)blocks, 256, 0, st>>>(xb, M, K, ldb, nseg, s, sx, scale_in, xq);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if (write_codes) {
    if (bf16) sqk::rowsplit_kernel<true, 1, F8><<<(unsigned)blocks, 256, 0, st>>>(xb, M, K, ldb, nseg, s, sx, scale_in, xq);
    else sqk::rowsplit_kernel<false, 1, F8><<<(unsigned)blocks, 256, 0, st>>>(xb, M, K, ldb, nseg, s, sx, scale_in, xq);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  sqk::rowsplit_scales_kernel<F8><<<(unsigned)((M + 255) / 256), 256, 0, st>>>(sx, M, scale_in);
  return cudaGetLastError();
}

// One pass of the row quantiser: per-token scales (scale_in == NULL) or a given per-tensor
// scale; write_codes = 0 computes the per-token scales only.
static cudaError_t launch_rows(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                               const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                               const float* scale_in, int write_codes, cudaStream_t st) {
  const int64_t ldb = ldx * (bf16 ? 2 : 4);
  // LayerNorm rows of 12288 and 14336 and plain rows of 12288 below 4096 tokens: the
  // block-per-row group kernel with exactly 6 or 7 chunks per thread (two blocks per SM) beats
  // the chunk-pair kernel (one block of 8 warps per SM at 254 registers): 23.2 against 27.2 us
  // (LayerNorm) and 32.0 against 34.8 us (plain) at 2048 x 12288; plain rows of 14336 measured
  // 38.1 against 35.5 and stay on the chunk-pair kernel
  const bool long_few = bf16 && M < 4096 && (K == 12288 || (gamma_f && K == 14336));
  if (!long_few && rowpair_supported(K, bf16, false, M))  // chunk-pair rows of the model widths
    return launch_rowpair_quant(x, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, scale_in, write_codes, false, st);
  if (!gamma_f && K > 16384)  // long plain rows: split into segments, two passes
    return launch_rowsplit<false>(x, bf16, M, K, ldx, s, xq, sx, scale_in, write_codes, st);
  int pT = 0, pn = 0;
  if (K <= 8192 && rowpipe_shape(K, bf16, 4, &pT, &pn))  // staged rows, 4 chunks per thread
    return launch_rowpipe_quant(x, bf16, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, pT, pn, scale_in, write_codes,
                                st);
  int nch = 0;
  const int T = pick_row_threads(K, 8, &nch);
  if (T) {
    const int k = (int)K;
#define SQ_T(TT)                                                                                                    \
  if (T == TT)                                                                                                      \
    return bf16 ? launch_group_nch<true, TT>(nch, x, M, k, ldb, gamma_f, beta_f, s, eps, xq, sx, scale_in, write_codes, \
                                            st)                                                                     \
                : launch_group_nch<false, TT>(nch, x, M, k, ldb, gamma_f, beta_f, s, eps, xq, sx, scale_in,          \
                                             write_codes, st);
    SQ_T(32) SQ_T(64) SQ_T(128) SQ_T(256)
#undef SQ_T
  }
  const int need = (int)((K / 8 + sqk::ROW_THREADS - 1) / sqk::ROW_THREADS);
  const int k = (int)K;
#define SQ_LNQ_CASE(C)                                                                                          \
  if (need <= C)                                                                                                \
    return bf16 ? launch_lnq_t<true, C>(x, M, k, ldb, gamma_f, beta_f, s, eps, xq, sx, scale_in, write_codes, st) \
                : launch_lnq_t<false, (C > 16 ? 16 : C)>(x, M, k, ldb, gamma_f, beta_f, s, eps, xq, sx, scale_in,  \
                                                         write_codes, st);
  SQ_LNQ_CASE(1) SQ_LNQ_CASE(2) SQ_LNQ_CASE(4) SQ_LNQ_CASE(8) SQ_LNQ_CASE(16) SQ_LNQ_CASE(24) SQ_LNQ_CASE(32)
#undef SQ_LNQ_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_ln_smooth_quant(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx,
                                   const float* gamma_f, const float* beta_f, const float* s, float eps,
                                   int8_t* xq, float* sx, cudaStream_t st) {
  return launch_rows(x, bf16, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, nullptr, 1, st);
}

// FP8 variant (per-token E4M3 codes, scale = max / 448): the chunk-pair row kernels for the
// model widths, the block-per-row kernel otherwise.
cudaError_t launch_ln_smooth_quant_fp8(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx,
                                       const float* gamma_f, const float* beta_f, const float* s, float eps,
                                       uint8_t* xq, float* sx, cudaStream_t st) {
  int8_t* q = reinterpret_cast<int8_t*>(xq);
  if (rowpair_supported(K, bf16, false, M))
    return launch_rowpair_quant(x, M, K, ldx, gamma_f, beta_f, s, eps, q, sx, nullptr, 1, true, st);
  if (!gamma_f && K > 16384) return launch_rowsplit<true>(x, bf16, M, K, ldx, s, q, sx, nullptr, 1, st);
  const int64_t ldb = ldx * (bf16 ? 2 : 4);
  const int need = (int)((K / 8 + sqk::ROW_THREADS - 1) / sqk::ROW_THREADS);
  const int k = (int)K;
#define SQ_LNQ8_CASE(C)                                                                                      \
  if (need <= C)                                                                                             \
    return bf16 ? launch_lnq_t<true, C, true>(x, M, k, ldb, gamma_f, beta_f, s, eps, q, sx, nullptr, 1, st) \
                : launch_lnq_t<false, (C > 16 ? 16 : C), true>(x, M, k, ldb, gamma_f, beta_f, s, eps, q, sx,   \
                                                               nullptr, 1, st);
  SQ_LNQ8_CASE(1) SQ_LNQ8_CASE(2) SQ_LNQ8_CASE(4) SQ_LNQ8_CASE(8) SQ_LNQ8_CASE(16) SQ_LNQ8_CASE(24)
  SQ_LNQ8_CASE(32)
#undef SQ_LNQ8_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_ln_smooth_quant_per_tensor(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx,
                                              const float* gamma_f, const float* beta_f, const float* s, float eps,
                                              int static_scale, float* scale, int8_t* xq, float* sx,
                                              cudaStream_t st) {
  if (!static_scale) {
    // per-token scales into sx, then scale = max_m sx[m] (= max |y| / 127: division by 127
    // is monotone, so the max of the rounded quotients is the rounded quotient of the max)
    cudaError_t e = launch_rows(x, bf16, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, nullptr, 0, st);
    if (e != cudaSuccess) return e;
    sqk::max_of_vector_kernel<<<1, 1024, 0, st>>>(sx, M, scale);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_rows(x, bf16, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, scale, 1, st);
}

}  // namespace sqh

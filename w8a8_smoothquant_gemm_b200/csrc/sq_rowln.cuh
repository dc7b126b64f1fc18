// sq_rowln.cuh -- one thread block (256 threads) per activation row: row load into
// registers, LayerNorm statistics in a fixed reduction order, and the per-element
// LayerNorm output.
//
// LayerNorm ("4.2 W8A8 量化与 SmoothQuant", sec. 6): LN(x)_j = (x_j - mu)/sigma * gamma_j + beta_j.
// The pages give no epsilon or summation order; this library fixes them:
//   sigma = sqrt(var + eps), biased variance, two passes over the row;
//   the row is cut into 8-element chunks, chunk c belongs to thread c mod 256, each
//   thread adds its chunks' elements in increasing order into a binary32 partial that
//   starts at +0 (x for the mean, fma(d, d, acc) with d = x - mu for the variance);
//   partials combine pairwise inside each warp at shuffle distances 16, 8, 4, 2, 1, then
//   the 8 warp results at distances 4, 2, 1;  mu = sum / K,  var = sum / K,
//   rstd = 1 / sqrt(var + eps),  y_j = fma((x_j - mu) * rstd, gamma_j, beta_j).
// Every operation is a correctly rounded binary32 intrinsic, so the result does not
// depend on compiler contraction.
#pragma once

#include "sq_common.cuh"

namespace sqk {

constexpr int ROW_THREADS = 256;
constexpr int ROW_WARPS = ROW_THREADS / 32;

// Raw storage of up to MAXC 8-element chunks per thread: one 16-byte vector per chunk
// for bf16, two for fp32.
template <bool BF16, int MAXC>
struct RowChunks {
  static constexpr int VEC = BF16 ? 1 : 2;
  uint4 v[MAXC * VEC];

  __device__ __forceinline__ void load(const void* row, int nchunks) {
    const char* base = static_cast<const char*>(row);
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = threadIdx.x + i * ROW_THREADS;
      if (c < nchunks) {
#pragma unroll
        for (int h = 0; h < VEC; ++h) v[i * VEC + h] = ldg_stream16(base + (size_t)c * 16 * VEC + 16 * h);
      }
    }
  }

  __device__ __forceinline__ void get(int i, float f[8]) const {
    if (BF16) {
      unpack8_bf16(v[i], f);
    } else {
      const uint4 a = v[i * VEC], b = v[i * VEC + (VEC - 1)];
      f[0] = __uint_as_float(a.x); f[1] = __uint_as_float(a.y);
      f[2] = __uint_as_float(a.z); f[3] = __uint_as_float(a.w);
      f[4] = __uint_as_float(b.x); f[5] = __uint_as_float(b.y);
      f[6] = __uint_as_float(b.z); f[7] = __uint_as_float(b.w);
    }
  }
};

// Sum of one partial per thread in the fixed tree order; every thread gets the total.
// `red` is ROW_WARPS + 1 floats of shared memory owned by this call site.
__device__ __forceinline__ float block_sum_fixed(float p, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) p = __fadd_rn(p, __shfl_down_sync(0xffffffffu, p, o));
  if (lane == 0) red[warp] = p;
  __syncthreads();
  if (warp == 0) {
    float g = lane < ROW_WARPS ? red[lane] : 0.0f;
#pragma unroll
    for (int o = ROW_WARPS / 2; o >= 1; o >>= 1) g = __fadd_rn(g, __shfl_down_sync(0xffffffffu, g, o));
    if (lane == 0) red[ROW_WARPS] = g;
  }
  __syncthreads();
  return red[ROW_WARPS];
}

// Max over the block (order-free); every thread gets it.  `red`: ROW_WARPS + 1 floats.
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) red[warp] = v;
  __syncthreads();
  if (warp == 0) {
    float g = lane < ROW_WARPS ? red[lane] : 0.0f;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
    if (lane == 0) red[ROW_WARPS] = g;
  }
  __syncthreads();
  return red[ROW_WARPS];
}

// mu and rstd of the row held in `rc` (nchunks = K / 8).  `red` needs 2 * (ROW_WARPS + 1)
// floats of shared memory.
template <bool BF16, int MAXC>
__device__ __forceinline__ void row_stats(const RowChunks<BF16, MAXC>& rc, int nchunks, int K,
                                          float eps, float* red, float& mu, float& rstd) {
  float acc = 0.0f;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    if ((int)threadIdx.x + i * ROW_THREADS < nchunks) {
      float f[8];
      rc.get(i, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc = __fadd_rn(acc, f[e]);
    }
  }
  const float kf = (float)K;
  mu = __fdiv_rn(block_sum_fixed(acc, red), kf);
  float acc2 = 0.0f;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    if ((int)threadIdx.x + i * ROW_THREADS < nchunks) {
      float f[8];
      rc.get(i, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = __fsub_rn(f[e], mu);
        acc2 = __fmaf_rn(d, d, acc2);
      }
    }
  }
  const float var = __fdiv_rn(block_sum_fixed(acc2, red + ROW_WARPS + 1), kf);
  rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps)));
}

// y = fma((x - mu) * rstd, g, b) for the 8 elements of chunk c (gamma/beta read from
// global memory; beta may be NULL).
__device__ __forceinline__ void ln_chunk(const float x[8], float mu, float rstd, const float* gamma,
                                         const float* beta, int c, float y[8]) {
  const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma + (size_t)c * 8));
  const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma + (size_t)c * 8 + 4));
  float4 b0 = make_float4(0.f, 0.f, 0.f, 0.f), b1 = b0;
  if (beta) {
    b0 = __ldg(reinterpret_cast<const float4*>(beta + (size_t)c * 8));
    b1 = __ldg(reinterpret_cast<const float4*>(beta + (size_t)c * 8 + 4));
  }
  const float g[8] = {g0.x, g0.y, g0.z, g0.w, g1.x, g1.y, g1.z, g1.w};
  const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] = __fmaf_rn(__fmul_rn(__fsub_rn(x[e], mu), rstd), g[e], b[e]);
}

// y = x / s for the 8 elements of chunk c.
__device__ __forceinline__ void div_chunk(const float x[8], const float* s, int c, float y[8]) {
  const float4 s0 = __ldg(reinterpret_cast<const float4*>(s + (size_t)c * 8));
  const float4 s1 = __ldg(reinterpret_cast<const float4*>(s + (size_t)c * 8 + 4));
  const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
  for (int e = 0; e < 8; ++e) y[e] = __fdiv_rn(x[e], sv[e]);
}

// ============================================================================ row groups
// A row handled by a group of T threads (T in {32, 64, 128, 256}, 256 / T groups per block
// of 256 threads).  Thread t of the group owns chunks c = t + T m (m < NCH) and, for the
// fixed reduction order above, the 256 / T lanes t + T i: chunk c is lane c mod 256, i.e.
// partial i = m mod (256 / T), and each partial takes its chunks in increasing m.  The row
// is held as NCH * 8 floats in registers.

template <int T>
__device__ __forceinline__ void group_barrier(int gid) {
  if (T == 32) {
    __syncwarp();
  } else if (T == 256) {
    __syncthreads();
  } else {
    asm volatile("bar.sync %0, %1;" ::"r"(gid + 1), "r"(T) : "memory");
  }
}

// Fixed-order sum of the 256 lane partials p[0 .. 256/T) of this group; every thread of
// the group gets the total.  `red`: 8 floats of shared memory owned by this call site.
template <int T>
__device__ __forceinline__ float group_sum_fixed(const float* p, float* red, int t, int gid) {
  constexpr int P = 256 / T;
  const int lane = t & 31, w = t >> 5;
#pragma unroll
  for (int i = 0; i < P; ++i) {
    float x = p[i];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) x = __fadd_rn(x, __shfl_down_sync(0xffffffffu, x, o));
    if (lane == 0) red[(T / 32) * i + w] = x;  // 32-lane group (T i + 32 w) / 32
  }
  group_barrier<T>(gid);
  float g[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) g[i] = red[i];
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1)
#pragma unroll
    for (int i = 0; i < o; ++i) g[i] = __fadd_rn(g[i], g[i + o]);
  return g[0];
}

// Max over the group (order-free); every thread of the group gets it.  `red`: T/32 floats.
template <int T>
__device__ __forceinline__ float group_max(float v, float* red, int t, int gid) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (T == 32) return v;
  if ((t & 31) == 0) red[t >> 5] = v;
  group_barrier<T>(gid);
  float m = red[0];
#pragma unroll
  for (int i = 1; i < T / 32; ++i) m = fmaxf(m, red[i]);
  return m;
}

// Raw 16-byte vectors of the chunks a thread owns (for loads ahead of use).
template <bool BF16, int NCH>
struct RowRaw {
  static constexpr int VEC = BF16 ? 1 : 2;
  uint4 v[NCH * VEC];
  template <int T>
  __device__ __forceinline__ void load(const char* row, int nchunks, int t) {
#pragma unroll
    for (int m = 0; m < NCH; ++m) {
      const int c = t + T * m;
      if (c < nchunks) {
#pragma unroll
        for (int h = 0; h < VEC; ++h) v[m * VEC + h] = ldg_stream16(row + (size_t)c * 16 * VEC + 16 * h);
      }
    }
  }
  __device__ __forceinline__ void to_float(float* f) const {
#pragma unroll
    for (int m = 0; m < NCH; ++m) {
      if (BF16) {
        unpack8_bf16(v[m], f + m * 8);
      } else {
        const uint4 a = v[m * VEC], b = v[m * VEC + VEC - 1];
        f[m * 8 + 0] = __uint_as_float(a.x); f[m * 8 + 1] = __uint_as_float(a.y);
        f[m * 8 + 2] = __uint_as_float(a.z); f[m * 8 + 3] = __uint_as_float(a.w);
        f[m * 8 + 4] = __uint_as_float(b.x); f[m * 8 + 5] = __uint_as_float(b.y);
        f[m * 8 + 6] = __uint_as_float(b.z); f[m * 8 + 7] = __uint_as_float(b.w);
      }
    }
  }
};

// mu and rstd of the row v[] (chunks c = t + T m) in the fixed order.  red: 16 floats.
template <int T, int NCH>
__device__ __forceinline__ void group_row_stats(const float* v, int nchunks, int K, float eps, float* red, int t,
                                                int gid, float& mu, float& rstd) {
  constexpr int P = 256 / T;
  float p[P];
#pragma unroll
  for (int i = 0; i < P; ++i) p[i] = 0.0f;
#pragma unroll
  for (int m = 0; m < NCH; ++m)
    if (t + T * m < nchunks)
#pragma unroll
      for (int e = 0; e < 8; ++e) p[m % P] = __fadd_rn(p[m % P], v[m * 8 + e]);
  const float kf = (float)K;
  mu = __fdiv_rn(group_sum_fixed<T>(p, red, t, gid), kf);
#pragma unroll
  for (int i = 0; i < P; ++i) p[i] = 0.0f;
#pragma unroll
  for (int m = 0; m < NCH; ++m)
    if (t + T * m < nchunks)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = __fsub_rn(v[m * 8 + e], mu);
        p[m % P] = __fmaf_rn(d, d, p[m % P]);
      }
  const float var = __fdiv_rn(group_sum_fixed<T>(p, red + 8, t, gid), kf);
  rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps)));
}

// As group_row_stats, but leaves d = x - mu in v[] (the LayerNorm output is then
// fma(d * rstd, gamma, beta)) and returns only rstd.
template <int T, int NCH>
__device__ __forceinline__ void group_row_stats_d(float* v, int nchunks, int K, float eps, float* red, int t, int gid,
                                                  float& rstd) {
  constexpr int P = 256 / T;
  float p[P];
#pragma unroll
  for (int i = 0; i < P; ++i) p[i] = 0.0f;
#pragma unroll
  for (int m = 0; m < NCH; ++m)
    if (t + T * m < nchunks)
#pragma unroll
      for (int e = 0; e < 8; ++e) p[m % P] = __fadd_rn(p[m % P], v[m * 8 + e]);
  const float kf = (float)K;
  const float mu = __fdiv_rn(group_sum_fixed<T>(p, red, t, gid), kf);
#pragma unroll
  for (int i = 0; i < P; ++i) p[i] = 0.0f;
#pragma unroll
  for (int m = 0; m < NCH; ++m)
    if (t + T * m < nchunks)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float d = __fsub_rn(v[m * 8 + e], mu);
        v[m * 8 + e] = d;
        p[m % P] = __fmaf_rn(d, d, p[m % P]);
      }
  const float var = __fdiv_rn(group_sum_fixed<T>(p, red + 8, t, gid), kf);
  rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps)));
}

}  // namespace sqk

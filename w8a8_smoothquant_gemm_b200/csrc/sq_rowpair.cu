// sq_rowpair.cu -- activation-row kernels for the row lengths of the model shapes
// (K = 8 T NCH exactly), written for instruction count: the same three modes as the
// staged row kernel of sq_rowpipe.cu --
//   LN_QUANT     fused LayerNorm (folded gamma' = gamma/s, beta' = beta/s) -> per-token INT8
//   PLAIN_QUANT  y = x / s (input from a previous GEMM)                     -> per-token INT8
//   LN_CALIB     per-channel absmax of LayerNorm(x) with the original gamma, beta
// ("4.2 W8A8 量化与 SmoothQuant", sec. 6 and 7.1; "量化：只压权重，与训练后量化（PTQ）",
// per-token activation quantisation), with the results of sq_rowpipe.cu bit for bit.
//
// Layout.  A row is handled by a group of T threads (one to eight warps).  Thread t
// owns the chunk pairs (c0, c1) = (2 T q + t, 2 T q + T + t), q < NCH / 2, and keeps
// element e of both chunks in one float2, so that every per-element step (the LayerNorm
// sums, its apply, the Markstein quotient, the rounding add) runs on packed binary32 pairs.
// Each half of a pair rounds exactly as the scalar operation would.
//
// Fixed reduction order (as in sq_rowln.cuh): chunk c belongs to virtual lane c mod 256, so
// c0 and c1 feed two different lane partials, and the float2 accumulator adds both lanes'
// elements in the order the lane itself would.  The 256 partials then combine in the fixed
// tree (offsets 16..1 inside each 32-lane group, then 4, 2, 1 across the 8 groups).  A warp
// holds 256 / T of those 32-lane groups, one per partial; the first levels of their trees
// run as a transposed butterfly (each exchange halves the groups a lane carries, and the
// lane keeps the half whose pair sums it finishes).  Floating-point addition is commutative,
// so computing p[t + o] + p[t] instead of p[t] + p[t + o] in the upper lane gives the same
// value, and every lane ends with exactly the value the canonical tree gives its group.
//
// Staging.  Each thread streams its own chunks of the next rows into an S-slot ring in
// shared memory with 16-byte cp.async (measured faster here than one bulk copy per row,
// which needs a poll and a group barrier per row); the per-channel vectors sit in
// shared memory in the pair order ([e/2][pair] float4s {v[c0][e], v[c1][e], v[c0][e+1],
// v[c1][e+1]}), so one conflict-free 16-byte read gives the operands of two packed steps.
#include <algorithm>

#include "sq_ptx.cuh"
#include "sq_rowln.cuh"


namespace sqk {

enum PairMode : int { PAIR_LN_QUANT = 0, PAIR_PLAIN_QUANT = 1, PAIR_LN_CALIB = 2 };

// Lane that holds the total of group i after the transposed butterfly over P groups (the
// exchange at distance 16 >> k decides bit (log2 P - 1 - k) of the group index).
template <int P>
__device__ __forceinline__ constexpr int pair_src_lane(int i) {
  return P == 8 ? ((i >> 2) & 1) * 16 + ((i >> 1) & 1) * 8 + (i & 1) * 4
       : P == 4 ? ((i >> 1) & 1) * 16 + (i & 1) * 8
                : (i & 1) * 16;
}

// v[i] is this lane's partial for 32-lane group i (position = lane).  Returns the group
// total of the canonical tree for group `idx`, which the butterfly assigns to this lane.
template <int P>
__device__ __forceinline__ float transposed_group_sums(float (&v)[P], int lane, int& idx) {
  idx = 0;
  int o = 16;
#pragma unroll
  for (int n = P; n > 1; n >>= 1, o >>= 1) {
    const bool hi = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float keep = hi ? v[j + n / 2] : v[j];
      const float send = hi ? v[j] : v[j + n / 2];
      v[j] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, o));
    }
    idx = idx * 2 + (hi ? 1 : 0);
  }
  float s = v[0];
#pragma unroll
  for (; o >= 1; o >>= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, o));
  return s;
}

// Fixed-order sum of a row from this thread's packed lane partials (acc[k].x = partial 2k,
// acc[k].y = partial 2k + 1; partial i is virtual lane t + T i).  Every thread of the group
// gets the total.  `red`: 8 floats of shared memory owned by this call site (T > 32).
template <int T>
__device__ __forceinline__ float pair_sum_fixed(const float2* acc, float* red, int t, int gid) {
  constexpr int P = 256 / T;
  const int lane = t & 31, w = t >> 5;
  float v[P];
#pragma unroll
  for (int k = 0; k < P / 2; ++k) {
    v[2 * k] = acc[k].x;
    v[2 * k + 1] = acc[k].y;
  }
  int idx;
  const float s = transposed_group_sums<P>(v, lane, idx);
  float g[8];
  if (T == 32) {
#pragma unroll
    for (int i = 0; i < 8; ++i) g[i] = __shfl_sync(0xffffffffu, s, pair_src_lane<P>(i));
  } else {
    // this warp's groups are w + (T / 32) i; one lane per group publishes its total
    if ((lane & (32 / P - 1)) == 0) red[w + (T / 32) * idx] = s;
    group_barrier<T>(gid);
#pragma unroll
    for (int i = 0; i < 8; ++i) g[i] = red[i];
  }
#pragma unroll
  for (int o = 4; o >= 1; o >>= 1)
#pragma unroll
    for (int i = 0; i < o; ++i) g[i] = __fadd_rn(g[i], g[i + o]);
  return g[0];
}

// RN(s / K) for the row length K: a multiplication by 2^-k when K = 2^k (the same exact
// quotient, rounded once), else the correctly rounded division.
template <int K>
__device__ __forceinline__ float div_by_len(float s) {
  if constexpr ((K & (K - 1)) == 0) return __fmul_rn(s, 1.0f / (float)K);
  else return __fdiv_rn(s, (float)K);
}

// Max over the group (order-free).  `red`: T / 32 floats (T > 32).
template <int T>
__device__ __forceinline__ float pair_group_max(float m, float* red, int t, int gid) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (T == 32) return m;
  if ((t & 31) == 0) red[t >> 5] = m;
  group_barrier<T>(gid);
  float r = red[0];
#pragma unroll
  for (int i = 1; i < T / 32; ++i) r = fmaxf(r, red[i]);
  return r;
}

// E4M3 codes of the 16 values of one chunk pair (the FP8 variant): the same quotient with the
// dividend's sign kept on zero results, then the saturating conversion; c0 gets the .x halves.
__device__ __forceinline__ void pair_codes_e4m3(const float2* v, const SharedDivisor& d, uint2& c0, uint2& c1) {
  float lo[8], hi[8];
  if (d.fast) {
    if (d.y == 0.0f) {  // zero scale: +0 codes
      c0 = c1 = make_uint2(0u, 0u);
      return;
    }
    const float2 rc = make_float2(d.y, d.y), nb = make_float2(-d.b, -d.b);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float2 qq = markstein2(v[e], rc, nb);
      lo[e] = with_sign_of(qq.x, v[e].x);
      hi[e] = with_sign_of(qq.y, v[e].y);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      lo[e] = d.div(v[e].x);
      hi[e] = d.div(v[e].y);
    }
  }
  c0 = make_uint2(e4m3x4(lo[0], lo[1], lo[2], lo[3]), e4m3x4(lo[4], lo[5], lo[6], lo[7]));
  c1 = make_uint2(e4m3x4(hi[0], hi[1], hi[2], hi[3]), e4m3x4(hi[4], hi[5], hi[6], hi[7]));
}

// Codes of the 16 values of one chunk pair with a shared scale (Markstein quotient and the
// rounding add of sq_common.cuh, on packed pairs); c0 gets the .x halves, c1 the .y halves.
template <bool CLAMP>
__device__ __forceinline__ void pair_codes_fast(const float2* v, const SharedDivisor& d, uint2& c0, uint2& c1) {
  const float2 rc = make_float2(d.y, d.y), nb = make_float2(-d.b, -d.b);
  const float2 magic = make_float2(12582912.0f, 12582912.0f);
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    float2 qq = markstein2(v[e], rc, nb);
    if (CLAMP) qq = make_float2(fminf(fmaxf(qq.x, -127.0f), 127.0f), fminf(fmaxf(qq.y, -127.0f), 127.0f));
    const float2 s = __fadd2_rn(qq, magic);
    lo[e] = __float_as_uint(s.x);
    hi[e] = __float_as_uint(s.y);
  }
  c0 = make_uint2(pack4_low_bytes(lo[0], lo[1], lo[2], lo[3]), pack4_low_bytes(lo[4], lo[5], lo[6], lo[7]));
  c1 = make_uint2(pack4_low_bytes(hi[0], hi[1], hi[2], hi[3]), pack4_low_bytes(hi[4], hi[5], hi[6], hi[7]));
}

// The same with a correctly rounded division (a scale outside Markstein's range), clamped.
__device__ __forceinline__ void pair_codes_slow(const float2* v, const SharedDivisor& d, uint2& c0, uint2& c1) {
  uint32_t lo[8], hi[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float a = fminf(fmaxf(d.div(v[e].x), -127.0f), 127.0f);
    const float b = fminf(fmaxf(d.div(v[e].y), -127.0f), 127.0f);
    lo[e] = __float_as_uint(__fadd_rn(a, 12582912.0f));
    hi[e] = __float_as_uint(__fadd_rn(b, 12582912.0f));
  }
  c0 = make_uint2(pack4_low_bytes(lo[0], lo[1], lo[2], lo[3]), pack4_low_bytes(lo[4], lo[5], lo[6], lo[7]));
  c1 = make_uint2(pack4_low_bytes(hi[0], hi[1], hi[2], hi[3]), pack4_low_bytes(hi[4], hi[5], hi[6], hi[7]));
}

// bf16 rows of K = 8 T NCH elements.  vec_a / vec_b: gamma' / beta' (LN_QUANT, beta' may be
// NULL), s / unused (PLAIN_QUANT), gamma / beta (LN_CALIB).  scale_in: the per-tensor scale
// (codes clamp), else per-token scales; write_codes = 0 writes sx only.  F8: E4M3 codes with
// scale = max / 448 (the FP8 variant; per-token scales only).
template <int T, int NCH, int W, int S, int MODE, bool F8 = false>
__global__ void __launch_bounds__(32 * W, 1)
rowpair_kernel(const char* __restrict__ x, int64_t M, int64_t ld_bytes, const float* __restrict__ vec_a,
               const float* __restrict__ vec_b, float eps, int8_t* __restrict__ xq, float* __restrict__ sx,
               float* __restrict__ out, const float* __restrict__ scale_in, int write_codes) {
  allow_dependent_launch();
  constexpr int NT = 32 * W;
  constexpr int G = NT / T;
  constexpr int P = 256 / T;
  constexpr bool ODD = NCH % 2 != 0;  // the last pair has no second chunk (plain mode only)
  constexpr int NQ = (NCH + 1) / 2;
  constexpr int NCHUNK = T * NCH;
  constexpr int K = NCHUNK * 8;
  constexpr int ROWB = K * 2;
  constexpr int NPAIR = NQ * T;
  constexpr bool LN = MODE != PAIR_PLAIN_QUANT;
  // the LayerNorm modes need two lane partials per thread (T <= 128, chunks in pairs); plain
  // rows have no reduction order and take 256-thread groups and an odd chunk count too
  static_assert(T >= 32 && NT % T == 0 && (LN ? (T <= 128 && !ODD) : T <= 256), "row group shape");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  float4* va = reinterpret_cast<float4*>(sm);  // [4][NPAIR]: gamma' | -s | gamma
  float4* vb = va + 4 * NPAIR;                 // [4][NPAIR]: beta'  | RN(1/s) | beta
  uint8_t* ring = reinterpret_cast<uint8_t*>(vb + 4 * NPAIR);  // [G][S][ROWB]
  __shared__ float red[G][24];

  const int gid = threadIdx.x / T, t = threadIdx.x % T;

  int slow = 0;
  {
    float* fa = reinterpret_cast<float*>(va);
    float* fb = reinterpret_cast<float*>(vb);
    for (int j = threadIdx.x; j < K; j += NT) {
      const int c = j >> 3, e = j & 7;
      const int rr = c % (2 * T);
      const int u = (c / (2 * T)) * T + rr % T;
      const int at = ((e >> 1) * NPAIR + u) * 4 + (e & 1) * 2 + rr / T;
      const float a = vec_a[j];
      if (MODE == PAIR_PLAIN_QUANT) {
        const bool fast = fabsf(a) >= 0x1p-90f && fabsf(a) <= 0x1p+90f;
        slow |= !fast;
        fa[at] = -a;
        fb[at] = fast ? __frcp_rn(a) : 0.0f;
      } else {
        fa[at] = a;
        fb[at] = vec_b ? vec_b[j] : 0.0f;
      }
    }
  }
  const bool all_fast = !__syncthreads_or(slow);

  uint8_t* gring = ring + (size_t)gid * S * ROWB;
  const int64_t rstep = (int64_t)gridDim.x * G;
  const int64_t r0 = (int64_t)blockIdx.x * G + gid;
  // Every thread copies exactly the chunks it reads (16-byte cp.async, one commit group per
  // row, empty past the last row), so a slot needs no barrier between its copy and its use,
  // and it is refilled as soon as its thread has moved the row into registers.
  auto issue = [&](int slot, int64_t r) {
    if (r < M) {
      const uint32_t dst = smem_u32(gring + (size_t)slot * ROWB);
      const char* src = x + r * ld_bytes;
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          if (ODD && q == NQ - 1 && h == 1) continue;  // no such chunk
          const int c = 2 * T * q + h * T + t;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst + c * 16), "l"(src + (size_t)c * 16)
                       : "memory");
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  for (int k = 0; k < S; ++k) issue(k, r0 + k * rstep);

  float2 cm[MODE == PAIR_LN_CALIB ? NQ * 8 : 1];
  if (MODE == PAIR_LN_CALIB) {
#pragma unroll
    for (int i = 0; i < NQ * 8; ++i) cm[i] = make_float2(0.0f, 0.0f);
  }

  int64_t it = 0;
  for (int64_t r = r0; r < M; r += rstep, ++it) {
    const int slot = (int)(it % S);
    asm volatile("cp.async.wait_group %0;" ::"n"(S - 1) : "memory");  // this row's copies
    const uint8_t* rowp = gring + (size_t)slot * ROWB;

    float2 v[NQ][8];  // v[q][e] = element e of chunks (2 T q + t, 2 T q + T + t)
#pragma unroll
    for (int q = 0; q < NQ; ++q) {
      const uint4 a = *reinterpret_cast<const uint4*>(rowp + (size_t)(2 * T * q + t) * 16);
      const uint4 b = (ODD && q == NQ - 1) ? make_uint4(0u, 0u, 0u, 0u)
                                           : *reinterpret_cast<const uint4*>(rowp + (size_t)(2 * T * q + T + t) * 16);
      v[q][0] = make_float2(bf16lo(a.x), bf16lo(b.x));
      v[q][1] = make_float2(bf16hi(a.x), bf16hi(b.x));
      v[q][2] = make_float2(bf16lo(a.y), bf16lo(b.y));
      v[q][3] = make_float2(bf16hi(a.y), bf16hi(b.y));
      v[q][4] = make_float2(bf16lo(a.z), bf16lo(b.z));
      v[q][5] = make_float2(bf16hi(a.z), bf16hi(b.z));
      v[q][6] = make_float2(bf16lo(a.w), bf16lo(b.w));
      v[q][7] = make_float2(bf16hi(a.w), bf16hi(b.w));
    }

    if constexpr (LN) {
      // mean: lane partials in increasing chunk and element order
      float2 acc[P / 2];
#pragma unroll
      for (int k = 0; k < P / 2; ++k) acc[k] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[q % (P / 2)] = __fadd2_rn(acc[q % (P / 2)], v[q][e]);
      const float mu = div_by_len<K>(pair_sum_fixed<T>(acc, red[gid], t, gid));
      issue(slot, r + S * rstep);  // this thread's share of the slot is in registers
      // variance of d = x - mu (d kept in v)
      const float2 nmu = make_float2(-mu, -mu);
#pragma unroll
      for (int k = 0; k < P / 2; ++k) acc[k] = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 d = __fadd2_rn(v[q][e], nmu);
          v[q][e] = d;
          acc[q % (P / 2)] = __ffma2_rn(d, d, acc[q % (P / 2)]);
        }
      const float var = div_by_len<K>(pair_sum_fixed<T>(acc, red[gid] + 8, t, gid));
      const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(var, eps)));
      const float2 rs2 = make_float2(rstd, rstd);
      // y = fma(d * rstd, gamma, beta)
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float4 g = va[h * NPAIR + q * T + t];
          const float4 b = vb[h * NPAIR + q * T + t];
          v[q][2 * h] = __ffma2_rn(__fmul2_rn(v[q][2 * h], rs2), make_float2(g.x, g.y), make_float2(b.x, b.y));
          v[q][2 * h + 1] =
              __ffma2_rn(__fmul2_rn(v[q][2 * h + 1], rs2), make_float2(g.z, g.w), make_float2(b.z, b.w));
        }
    } else if (all_fast) {
      // y = x / s: Markstein with the per-channel RN(1/s) (q = RN(x y), r = x - s q exact,
      // RN(q + r y) = RN(x / s))
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float4 ns = va[h * NPAIR + q * T + t];
          const float4 rs = vb[h * NPAIR + q * T + t];
          const float2 r01 = make_float2(rs.x, rs.y), r23 = make_float2(rs.z, rs.w);
          const float2 x01 = v[q][2 * h], x23 = v[q][2 * h + 1];
          v[q][2 * h] = markstein2(x01, r01, make_float2(ns.x, ns.y));
          v[q][2 * h + 1] = markstein2(x23, r23, make_float2(ns.z, ns.w));
          if (F8) {  // RN(-0 / s) = -0, which Markstein's correction turns into +0; E4M3 keeps the sign
            v[q][2 * h] = make_float2(with_sign_of(v[q][2 * h].x, x01.x), with_sign_of(v[q][2 * h].y, x01.y));
            v[q][2 * h + 1] = make_float2(with_sign_of(v[q][2 * h + 1].x, x23.x), with_sign_of(v[q][2 * h + 1].y, x23.y));
          }
        }
    } else {  // a divisor outside Markstein's range somewhere in s
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float4 ns = va[h * NPAIR + q * T + t];
          v[q][2 * h] = make_float2(__fdiv_rn(v[q][2 * h].x, -ns.x), __fdiv_rn(v[q][2 * h].y, -ns.y));
          v[q][2 * h + 1] = make_float2(__fdiv_rn(v[q][2 * h + 1].x, -ns.z), __fdiv_rn(v[q][2 * h + 1].y, -ns.w));
        }
    }

    if (ODD) {  // the missing chunk of the last pair (its factors in shared memory are not set)
#pragma unroll
      for (int e = 0; e < 8; ++e) v[NQ - 1][e].y = 0.0f;
    }

    if (MODE == PAIR_LN_CALIB) {
#pragma unroll
      for (int q = 0; q < NQ; ++q)
#pragma unroll
        for (int e = 0; e < 8; ++e)
          cm[q * 8 + e] = make_float2(fmaxf(cm[q * 8 + e].x, fabsf(v[q][e].x)), fmaxf(cm[q * 8 + e].y, fabsf(v[q][e].y)));
      continue;
    }

    // ---- per-token quantisation
    float am[4] = {0.0f, 0.0f, 0.0f, 0.0f};  // independent max chains
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int e = 0; e < 8; ++e) am[e & 3] = fmax3(am[e & 3], fabsf(v[q][e].x), fabsf(v[q][e].y));
    float amax = fmax3(am[0], am[1], fmaxf(am[2], am[3]));
    amax = pair_group_max<T>(amax, red[gid] + 16, t, gid);
    if (!LN) issue(slot, r + S * rstep);  // this thread's share of the slot is in registers
    const float scale = scale_in ? __ldg(scale_in) : __fdiv_rn(amax, F8 ? 448.0f : 127.0f);
    if (t == 0) sx[r] = scale;
    if (F8) {
      const SharedDivisor d(scale);
      uint2* q0 = reinterpret_cast<uint2*>(xq + r * (int64_t)K) + t;
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        uint2 c0, c1;
        pair_codes_e4m3(v[q], d, c0, c1);
        q0[2 * T * q] = c0;
        if (!ODD || q < NQ - 1) q0[2 * T * q + T] = c1;
      }
    } else if (write_codes) {
      const SharedDivisor d(scale);
      const bool clamp = scale_in != nullptr;
      int8_t* qrow = xq + r * (int64_t)K;
      uint2* q0 = reinterpret_cast<uint2*>(qrow) + t;
      uint2 c0, c1;
      if (d.fast && !clamp) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          pair_codes_fast<false>(v[q], d, c0, c1);
          q0[2 * T * q] = c0;
          if (!ODD || q < NQ - 1) q0[2 * T * q + T] = c1;
        }
      } else if (d.fast) {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          pair_codes_fast<true>(v[q], d, c0, c1);
          q0[2 * T * q] = c0;
          if (!ODD || q < NQ - 1) q0[2 * T * q + T] = c1;
        }
      } else {
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          pair_codes_slow(v[q], d, c0, c1);
          q0[2 * T * q] = c0;
          if (!ODD || q < NQ - 1) q0[2 * T * q + T] = c1;
        }
      }
    }
  }

  if (MODE == PAIR_LN_CALIB) {
    // merge the groups' column maxima through shared memory (the ring is idle now), then
    // one atomicMax per column per block
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    float* scratch = reinterpret_cast<float*>(ring);  // [G][K]
#pragma unroll
    for (int q = 0; q < NQ; ++q)
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        scratch[gid * K + (2 * T * q + t) * 8 + e] = cm[q * 8 + e].x;
        scratch[gid * K + (2 * T * q + T + t) * 8 + e] = cm[q * 8 + e].y;
      }
    __syncthreads();
    if ((int64_t)blockIdx.x * G < M)
      for (int j = threadIdx.x; j < K; j += NT) {
        float mx = scratch[j];
#pragma unroll
        for (int g = 1; g < G; ++g) mx = fmaxf(mx, scratch[g * K + j]);
        atomic_max_nonneg(out + j, mx);
      }
  }
}

}  // namespace sqk

namespace sqh {

// Shared memory of one block: the two per-channel vectors (npair pairs of 8-value chunks each)
// and the rings.
static constexpr size_t rowpair_smem(int K, int npair, int G, int S) {
  return 128 + (size_t)npair * 128 + (size_t)G * S * K * 2;
}

template <int T, int NCH, int W, int S, int MODE, bool F8>
static cudaError_t launch_rowpair(const void* x, int64_t M, int64_t ld_bytes, const float* va, const float* vb,
                                  float eps, int8_t* xq, float* sx, float* out, const float* scale_in,
                                  int write_codes, cudaStream_t st) {
  constexpr int G = 32 * W / T;
  constexpr size_t smem = rowpair_smem(8 * T * NCH, (NCH + 1) / 2 * T, G, S);
  static_assert(smem + sizeof(float) * G * 24 <= 227 * 1024, "block exceeds the shared memory of an SM");
  auto kern = sqk::rowpair_kernel<T, NCH, W, S, MODE, F8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 32 * W, smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (M + G - 1) / G;
  const int64_t grid = std::min<int64_t>(blocks, (int64_t)num_sms() * std::max(per_sm, 1));
  kern<<<(unsigned)grid, 32 * W, smem, st>>>((const char*)x, M, ld_bytes, va, vb, eps, xq, sx, out, scale_in,
                                             write_codes);
  return cudaGetLastError();
}

// Row lengths with a chunk-pair kernel (bf16 rows only).  Quantisers: K in {512, 1024, 2048,
// 4096, 8192, 12288, 14336}; calibration (whose running maxima also live in registers):
// K in {512, 1024, 2048, 4096, 8192}.  Below 1024 rows the staged kernel of sq_rowpipe.cu
// runs instead: with few rows per group, the per-row latency outweighs the instruction savings.
bool rowpair_supported(int64_t K, bool bf16, bool calib, int64_t rows) {
  if (!bf16 || rows < 1024) return false;
  switch (K) {
    case 512: case 1024: case 2048: case 4096: case 8192: return true;
    case 12288: case 14336: return !calib;
    default: return false;
  }
}

template <int MODE, bool F8 = false>
static cudaError_t launch_rowpair_mode(int64_t K, const void* x, int64_t M, int64_t ldb, const float* va,
                                       const float* vb, float eps, int8_t* xq, float* sx, float* out,
                                       const float* scale_in, int write_codes, cudaStream_t st) {
  constexpr bool CAL = MODE == sqk::PAIR_LN_CALIB;
#define SQ_PAIR(T, NCH, W, S) \
  launch_rowpair<T, NCH, W, S, MODE, F8>(x, M, ldb, va, vb, eps, xq, sx, out, scale_in, write_codes, st)
  switch (K) {
    case 512: return SQ_PAIR(32, 2, 16, 2);
    case 1024: return SQ_PAIR(64, 2, 16, 2);
    case 2048: return SQ_PAIR(64, 4, 16, 2);
    default: break;
  }
  if constexpr (CAL) {
    // K = 4096: four-warp groups (124 registers, 16 warps per SM) beat two-warp groups with
    // twice the chunks (250 registers, 8 warps per SM): measured 135 against 143 us at 65536 rows
    if (K == 4096) return SQ_PAIR(128, 4, 16, 2);
    if (K == 8192) return SQ_PAIR(128, 8, 8, 2);
  } else {
    if (K == 4096) return SQ_PAIR(64, 8, 16, 2);
    if (K == 8192) {
      // plain rows: four-warp groups with one ring slot (126 registers, 16 warps per SM)
      // beat two-warp groups (255 registers, 8 warps per SM): 51 against 55 us at 8192 rows
      if constexpr (MODE == sqk::PAIR_PLAIN_QUANT) return SQ_PAIR(128, 8, 16, 1);
      return SQ_PAIR(64, 16, 8, 2);
    }
    if (K == 12288) return SQ_PAIR(128, 12, 8, 2);
    if (K == 14336) {
      // plain rows (no reduction order): below ~4k rows, 256-thread groups (an odd 7 chunks
      // per thread, 16 warps per SM, one ring slot) beat two-warp groups (8 warps per SM);
      // measured 37 against 44 us at 2048 rows, 105 against 91 us at 8192
      if constexpr (MODE == sqk::PAIR_PLAIN_QUANT) {
        if (M < 4096) return SQ_PAIR(256, 7, 16, 1);
      }
      return SQ_PAIR(128, 14, 8, 2);
    }
  }
#undef SQ_PAIR
  return cudaErrorInvalidValue;
}

cudaError_t launch_rowpair_quant(const void* x, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                                 const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                                 const float* scale_in, int write_codes, bool f8, cudaStream_t st) {
  const int64_t ldb = ldx * 2;
  if (f8) {
    if (gamma_f)
      return launch_rowpair_mode<sqk::PAIR_LN_QUANT, true>(K, x, M, ldb, gamma_f, beta_f, eps, xq, sx, nullptr,
                                                           nullptr, 1, st);
    return launch_rowpair_mode<sqk::PAIR_PLAIN_QUANT, true>(K, x, M, ldb, s, nullptr, eps, xq, sx, nullptr, nullptr,
                                                            1, st);
  }
  if (gamma_f)
    return launch_rowpair_mode<sqk::PAIR_LN_QUANT>(K, x, M, ldb, gamma_f, beta_f, eps, xq, sx, nullptr, scale_in,
                                                   write_codes, st);
  return launch_rowpair_mode<sqk::PAIR_PLAIN_QUANT>(K, x, M, ldb, s, nullptr, eps, xq, sx, nullptr, scale_in,
                                                    write_codes, st);
}

cudaError_t launch_rowpair_calib(const void* x, int64_t rows, int64_t K, int64_t ldx, const float* gamma,
                                 const float* beta, float eps, float* out, cudaStream_t st) {
  return launch_rowpair_mode<sqk::PAIR_LN_CALIB>(K, x, rows, ldx * 2, gamma, beta, eps, nullptr, nullptr, out,
                                                 nullptr, 1, st);
}

}  // namespace sqh

// sq_common.cuh -- device helpers shared by the sm_100a kernels of the W8A8 library.
//
// Numerics: every floating-point operation that decides a result (a code, a scale, a
// LayerNorm statistic) is written with an explicit round-to-nearest intrinsic, so the
// compiler cannot fuse or reorder it (the library is also built with --fmad=false).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sq_w8a8.h"

namespace sqk {

// Device-side diagnostics (one per device, defined next to the GEMM): the error word that a
// kernel whose bounded wait ran out ORs its code into (read with sq_device_error()), and the
// limit of those waits (sq_set_wait_limit(); 0 makes every wait run out at once).  Kernels in
// other files get the address of `error` and read the limit beside it.
struct DeviceDiag {
  unsigned int error;
  unsigned int reserved;
  unsigned long long wait_limit_ns;
};

__device__ __forceinline__ unsigned long long wait_limit(const unsigned int* err) {
  return reinterpret_cast<const volatile DeviceDiag*>(err)->wait_limit_ns;
}

// Limit of the waits that let copies already issued land before a kernel that gave up leaves.
constexpr unsigned long long DRAIN_NS = 100ull * 1000 * 1000;

enum : unsigned int {
  ERR_GEMM_PRODUCER_WAIT = 1u << 0,
  ERR_GEMM_MMA_WAIT = 1u << 1,
  ERR_GEMM_EPILOGUE_WAIT = 1u << 2,
  ERR_FOLD_TMA_WAIT = 1u << 3,
  ERR_ROW_TMA_WAIT = 1u << 4,
};

// max(a, b, c) in one instruction (three-operand max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// bf16 bits -> fp32 (exact widening).
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// 8 consecutive elements as fp32 from one 16-byte bf16 vector.
__device__ __forceinline__ void unpack8_bf16(const uint4 v, float f[8]) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x);
  f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z);
  f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}

// Symmetric INT8 code: clamp(rne(v / scale), -127, 127); scale 0 -> 0.
__device__ __forceinline__ int quant_code(float v, float scale) {
  if (scale == 0.0f) return 0;
  int q = __float2int_rn(__fdiv_rn(v, scale));
  return max(-127, min(127, q));
}

// Division by a divisor shared by many dividends (a per-row or per-column scale).
// Markstein's theorem (P. Markstein, IBM J. Res. Dev. 34(1), 1990; Muller et al., Handbook
// of Floating-Point Arithmetic, sec. on division with FMA): with y = RN(1/b) and
// q = RN(a * y), the remainder r = a - b q is exact under FMA and RN(q + r y) is the
// correctly rounded a / b, barring underflow or overflow of the intermediates.
struct SharedDivisor {
  float b, y;
  bool fast;  // b is far from the subnormal range, so the intermediates stay normal
  // A zero divisor (all-zero row or column) is turned into "multiply by 0", so every code
  // of that row or column is 0, as the quantiser defines.
  __device__ __forceinline__ explicit SharedDivisor(float b_) : b(b_) {
    if (b_ == 0.0f) {
      b = 1.0f;
      y = 0.0f;
      fast = true;
      return;
    }
    fast = fabsf(b_) >= 0x1p-90f && fabsf(b_) <= 0x1p+90f;
    y = fast ? __frcp_rn(b_) : 0.0f;
  }
  __device__ __forceinline__ float div(float a) const {
    if (!fast) return __fdiv_rn(a, b);
    return div_fast(a);
  }
  // Markstein quotient only; valid when `fast` (callers branch once, outside their loops).
  __device__ __forceinline__ float div_fast(float a) const {
    const float q = __fmul_rn(a, y);
    const float r = __fmaf_rn(-q, b, a);
    return __fmaf_rn(r, y, q);
  }
};

// The same quotient on a packed binary32 pair, each half with its own divisor: rc holds the
// two correctly rounded reciprocals, nb the two negated divisors.  Each half rounds exactly as
// SharedDivisor::div_fast does.
__device__ __forceinline__ float2 markstein2(float2 a, float2 rc, float2 nb) {
  const float2 q = __fmul2_rn(a, rc);
  const float2 r = __ffma2_rn(q, nb, a);
  return __ffma2_rn(r, rc, q);
}

// Code of v with a shared scale, returned in the low byte of a 32-bit word: the
// correctly rounded quotient q = v / scale satisfies |q| <= 127 (1 + 2^-23) because
// |v| <= absmax and scale = RN(absmax / 127), so adding 1.5 * 2^23 rounds q to the nearest
// integer, ties to even (the float grid has spacing 1 there), and leaves rne(q) mod 256 in
// the low byte of the sum's bit pattern.  The clamp to [-127, 127] can never bind.
// A zero scale gives code 0 (see SharedDivisor).
__device__ __forceinline__ uint32_t code_bits(float v, const SharedDivisor& d) {
  return __float_as_uint(__fadd_rn(d.div(v), 12582912.0f));
}
__device__ __forceinline__ uint32_t code_bits_fast(float v, const SharedDivisor& d) {
  return __float_as_uint(__fadd_rn(d.div_fast(v), 12582912.0f));
}

// Low bytes of four words -> one packed word (first argument in the low byte).
__device__ __forceinline__ uint32_t pack4_low_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  return __byte_perm(__byte_perm(a, b, 0x0040), __byte_perm(c, d, 0x0040), 0x5410);
}

// Codes of 8 values (one chunk) packed into 8 bytes; FAST selects the Markstein-only path,
// evaluated two lanes at a time with packed binary32 arithmetic (each half rounds exactly
// as the scalar operation would).  CLAMP bounds the quotient to [-127, 127] first, which a
// scale that did not come from this data's own absmax (a calibrated per-tensor scale) needs.
template <bool FAST, bool CLAMP = false>
__device__ __forceinline__ uint2 pack8_codes(const float* y, const SharedDivisor& d) {
  uint32_t c[8];
  if (FAST) {
    const float2 rc = make_float2(d.y, d.y), nb = make_float2(-d.b, -d.b);
    const float2 magic = make_float2(12582912.0f, 12582912.0f);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      float2 qq = markstein2(make_float2(y[e], y[e + 1]), rc, nb);
      if (CLAMP) qq = make_float2(fminf(fmaxf(qq.x, -127.0f), 127.0f), fminf(fmaxf(qq.y, -127.0f), 127.0f));
      const float2 t = __fadd2_rn(qq, magic);
      c[e] = __float_as_uint(t.x);
      c[e + 1] = __float_as_uint(t.y);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float q = d.div(y[e]);
      if (CLAMP) q = fminf(fmaxf(q, -127.0f), 127.0f);
      c[e] = __float_as_uint(__fadd_rn(q, 12582912.0f));
    }
  }
  return make_uint2(pack4_low_bytes(c[0], c[1], c[2], c[3]), pack4_low_bytes(c[4], c[5], c[6], c[7]));
}

// ---------------------------------------------------------------------------- FP8 codes
// The FP8 variant of the method uses E4M3 codes (OCP 8-bit floating point, OFP8: bias 7,
// 3 mantissa bits, largest finite 448) with scale = max|.| / 448; the code of v is E4M3 of
// the correctly rounded quotient RN(v / scale), nearest even, saturating.

// E4M3 codes of four binary32 values, first argument in the low byte (the PTX conversion
// puts its first source operand in the upper byte of each pair).
__device__ __forceinline__ uint32_t e4m3x4(float a, float b, float c, float d) {
  uint32_t r;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
      "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
      "mov.b32 %0, {lo, hi};\n\t}"
      : "=r"(r)
      : "f"(a), "f"(b), "f"(c), "f"(d));
  return r;
}

// E4M3 code (byte value) of v with a scale: E4M3 of the correctly rounded RN(v / scale);
// scale 0 -> +0.
__device__ __forceinline__ int e4m3_code(float v, float scale) {
  if (scale == 0.0f) return 0;
  return (int)(e4m3x4(__fdiv_rn(v, scale), 0.0f, 0.0f, 0.0f) & 0xffu);
}

// The quotient with the dividend's sign: Markstein's correction step turns RN(-0 / b) = -0
// into +0, which E4M3 (unlike an integer code) tells apart.
__device__ __forceinline__ float with_sign_of(float q, float v) { return copysignf(q, v); }

// E4M3 codes of 8 values (one chunk) with a shared scale; a zero scale (all-zero row or
// column) gives +0 codes.
template <bool FAST>
__device__ __forceinline__ uint2 pack8_e4m3(const float* y, const SharedDivisor& d) {
  if (d.fast && d.y == 0.0f) return make_uint2(0u, 0u);  // zero scale
  float q[8];
  if (FAST) {
    const float2 rc = make_float2(d.y, d.y), nb = make_float2(-d.b, -d.b);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float2 qq = markstein2(make_float2(y[e], y[e + 1]), rc, nb);
      q[e] = with_sign_of(qq.x, y[e]);
      q[e + 1] = with_sign_of(qq.y, y[e + 1]);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 8; ++e) q[e] = d.div(y[e]);  // correctly rounded division keeps the sign
  }
  return make_uint2(e4m3x4(q[0], q[1], q[2], q[3]), e4m3x4(q[4], q[5], q[6], q[7]));
}

// Writes the codes of NCH chunks (chunk m of this thread at c = t + T m) of one row.
template <int T, int NCH>
__device__ __forceinline__ void store_row_codes(const float* v, int t, int nchunks, float scale, bool clamp,
                                                int8_t* qrow) {
  const SharedDivisor d(scale);
  if (d.fast && !clamp) {
#pragma unroll
    for (int m = 0; m < NCH; ++m)
      if (t + T * m < nchunks) *reinterpret_cast<uint2*>(qrow + (int64_t)(t + T * m) * 8) = pack8_codes<true>(v + m * 8, d);
  } else if (d.fast) {
#pragma unroll
    for (int m = 0; m < NCH; ++m)
      if (t + T * m < nchunks)
        *reinterpret_cast<uint2*>(qrow + (int64_t)(t + T * m) * 8) = pack8_codes<true, true>(v + m * 8, d);
  } else {  // rare: a scale outside the fast range
#pragma unroll
    for (int m = 0; m < NCH; ++m)
      if (t + T * m < nchunks)
        *reinterpret_cast<uint2*>(qrow + (int64_t)(t + T * m) * 8) = pack8_codes<false, true>(v + m * 8, d);
  }
}

// Packs four codes (low byte first) into one 32-bit word.
__device__ __forceinline__ uint32_t pack4_s8(int a, int b, int c, int d) {
  return (uint32_t)(a & 0xff) | ((uint32_t)(b & 0xff) << 8) | ((uint32_t)(c & 0xff) << 16) |
         ((uint32_t)(d & 0xff) << 24);
}

// Streaming 16-byte load that does not allocate in L1.
__device__ __forceinline__ uint4 ldg_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Lets the next kernel on the stream start its set-up, if it was launched as a programmatic
// dependent (the GEMM is: it allocates TMEM, initialises its barriers and asks L2 for its first
// weight tiles, and reads nothing that this kernel writes before its griddepcontrol.wait, which
// returns once this grid has completed and its writes are visible).  The quantisers call it
// first thing, so that in decode the GEMM's weight stream starts while the activations are
// quantised.  No effect when the next kernel is an ordinary launch.
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Max of non-negative floats through their bit patterns (monotone for x >= +0).
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
  atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
}

}  // namespace sqk

// Host-side launch helpers (internal to the library; no C ABI).
namespace sqh {
int num_sms();                    // SM count of the current device (cached per device)
// cudaOccupancyMaxActiveClusters, cached per device, kernel and launch shape
cudaError_t max_active_clusters(const void* kern, const cudaLaunchConfig_t* cfg, int* clusters);
unsigned int* error_word_ptr();   // device address of the error word (current device)
}  // namespace sqh

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

// Codes OR-ed into the device-side error word (defined next to the GEMM, the only
// kernel with waits) when a bounded wait runs out; read with sq_device_error().
enum : unsigned int {
  ERR_GEMM_PRODUCER_WAIT = 1u << 0,
  ERR_GEMM_MMA_WAIT = 1u << 1,
  ERR_GEMM_EPILOGUE_WAIT = 1u << 2,
};

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

// Max of non-negative floats through their bit patterns (monotone for x >= +0).
__device__ __forceinline__ void atomic_max_nonneg(float* addr, float v) {
  atomicMax(reinterpret_cast<int*>(addr), __float_as_int(v));
}

}  // namespace sqk

// Host-side launch helpers (internal to the library; no C ABI).
namespace sqh {
int num_sms();                 // SM count of the current device (cached per device)
size_t max_smem_optin();       // opt-in shared memory per block of the current device
}  // namespace sqh

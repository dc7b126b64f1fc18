// sq_selfcheck.cu -- on-device check of the shared-divisor quotient that every quantiser and
// the weight fold use in place of IEEE division.
//
// The per-token scale sx = max|y| / 127 (and the per-channel weight scale) divides every element
// of its row (column).  "SmoothQuant大模型平滑量化技术" (Python demo) defines the code as
// round(v / scale), so the quotient must be the correctly rounded one: a last-bit error can move
// a value across a rounding boundary and change its code.  The kernels compute it with one
// reciprocal per row and Markstein's correction step (SharedDivisor::div_fast and markstein2 in
// sq_common.cuh).  This kernel evaluates both forms for every (divisor, dividend) pair it is
// given and counts the pairs whose bits differ from RN(a / b).
#include <algorithm>

#include "sq_common.cuh"

namespace sqk {

constexpr int SELFCHECK_MAX_NA = 4096;

// One thread per divisor; the dividends are staged in shared memory.  counts[0]: mismatches of
// the scalar form (SharedDivisor::div), counts[1]: of the packed-pair form (markstein2, used when
// the divisor is in the fast range), counts[2]: pairs checked.  Zero divisors are skipped (the
// quantisers define that case as "all codes 0", not as a quotient).
__global__ void __launch_bounds__(256)
shared_divisor_check_kernel(const float* __restrict__ a, int na, const float* __restrict__ b, int64_t nb,
                            float* __restrict__ q, unsigned long long* __restrict__ counts) {
  __shared__ float sa[SELFCHECK_MAX_NA];
  for (int j = threadIdx.x; j < na; j += blockDim.x) sa[j] = a[j];
  __syncthreads();
  unsigned long long bad_s = 0, bad_p = 0, checked = 0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < nb; i += (int64_t)gridDim.x * blockDim.x) {
    const float bi = b[i];
    if (bi == 0.0f) continue;
    const SharedDivisor d(bi);
    const float2 rc = make_float2(d.y, d.y), nbv = make_float2(-d.b, -d.b);
    for (int j = 0; j < na; j += 2) {
      const float a0 = sa[j], a1 = sa[j + 1];
      const float r0 = __fdiv_rn(a0, bi), r1 = __fdiv_rn(a1, bi);
      const float s0 = d.div(a0), s1 = d.div(a1);
      const float2 p = d.fast ? markstein2(make_float2(a0, a1), rc, nbv) : make_float2(s0, s1);
      bad_s += (__float_as_uint(s0) != __float_as_uint(r0)) + (__float_as_uint(s1) != __float_as_uint(r1));
      bad_p += (__float_as_uint(p.x) != __float_as_uint(r0)) + (__float_as_uint(p.y) != __float_as_uint(r1));
      checked += 2;
      if (q) {
        q[i * na + j] = s0;
        q[i * na + j + 1] = s1;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    bad_s += __shfl_xor_sync(0xffffffffu, bad_s, o);
    bad_p += __shfl_xor_sync(0xffffffffu, bad_p, o);
    checked += __shfl_xor_sync(0xffffffffu, checked, o);
  }
  if ((threadIdx.x & 31) == 0) {
    if (bad_s) atomicAdd(counts, bad_s);
    if (bad_p) atomicAdd(counts + 1, bad_p);
    atomicAdd(counts + 2, checked);
  }
}

}  // namespace sqk

extern "C" sq_status sq_selfcheck_shared_divisor(const float* a, int64_t na, const float* b, int64_t nb, float* q,
                                                 unsigned long long* counts, void* stream) {
  if (na <= 0 || na > sqk::SELFCHECK_MAX_NA || na % 2 != 0 || nb < 0) return SQ_ERR_INVALID_ARG;
  if (!a || !counts || (nb > 0 && !b)) return SQ_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(counts) & 7u) != 0 || (reinterpret_cast<uintptr_t>(a) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(b) & 3u) != 0 || (reinterpret_cast<uintptr_t>(q) & 3u) != 0)
    return SQ_ERR_ALIGNMENT;
  if (nb == 0) return SQ_OK;
  const int64_t blocks = std::min<int64_t>((nb + 255) / 256, (int64_t)sqh::num_sms() * 8);
  sqk::shared_divisor_check_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(a, (int)na, b, nb,
                                                                                                   q, counts);
  return cudaGetLastError() == cudaSuccess ? SQ_OK : SQ_ERR_CUDA;
}

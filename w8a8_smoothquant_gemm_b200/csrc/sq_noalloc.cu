// sq_noalloc.cu -- a GEMM entry point for callers that cannot allocate device memory.
//
// sq_w8a8_gemm asks its caller for a workspace when it splits K across SMs (decode-sized
// M): the int32 partial sums of each K slice live there until the reduction kernel adds
// them up.  Some callers cannot provide one: a plug-in running inside a host program that
// owns all device memory through its own pool (a cudaMalloc would fail or break that
// program's accounting), or a latency-critical loop where cudaMalloc may synchronise the
// device.  sq_w8a8_gemm_noalloc serves them from a fixed scratch array that is part of
// the library image instead.
//
// The array is a file-scope __device__ variable of SQ_NOALLOC_SCRATCH_BYTES.  Every GPU
// that loads the library holds it until the process exits.  In host code its name is
// only a stand-in for the device variable, so its device address is looked up with
// cudaGetSymbolAddress once per device (with that device current) and that address is
// what the kernels receive.
#include <mutex>

#include "sq_common.cuh"

namespace sqh {
sq_status check_gemm_args(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M, int64_t N,
                          int64_t K, const void* y, sq_dtype ydt, int64_t ldy, bool* empty);
}

namespace sqh {
size_t gemm_workspace_size_min(int64_t M, int64_t N, int64_t K);
}  // namespace sqh

namespace {

static __device__ __align__(256) unsigned char g_gemm_scratch[SQ_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices];
cudaError_t g_scratch_status[kMaxDevices];
std::once_flag g_scratch_once[kMaxDevices];

// Device address of the scratch array on the current device (looked up on first use).
cudaError_t scratch_address(void** addr) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::call_once(g_scratch_once[dev], [dev] {
    void* p = nullptr;
    cudaError_t e = cudaGetSymbolAddress(&p, g_gemm_scratch);
    // the GEMM's split-work sums in the scratch must start at zero; every call leaves them at zero
    // again (a synchronous memset: this set-up precedes any stream capture)
    if (e == cudaSuccess) e = cudaMemset(p, 0, SQ_NOALLOC_SCRATCH_BYTES);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    g_scratch_status[dev] = e;
    g_scratch_addr[dev] = p;
  });
  if (g_scratch_status[dev] != cudaSuccess) return g_scratch_status[dev];
  *addr = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace

extern "C" sq_status sq_w8a8_gemm_noalloc(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw,
                                          int64_t M, int64_t N, int64_t K, void* y, sq_dtype ydt, int64_t ldy,
                                          void* stream) {
  // the same argument checks, in the same order, as sq_w8a8_gemm; the scratch size comes after
  bool empty = false;
  const sq_status st = sqh::check_gemm_args(xq, sx, wq, sw, M, N, K, y, ydt, ldy, &empty);
  if (st != SQ_OK || empty) return st;
  // the smallest workspace a launch of this shape runs with (the split tail of large CTA-pair
  // shapes is optional and not used here)
  const size_t need = sqh::gemm_workspace_size_min(M, N, K);
  if (need == 0) return sq_w8a8_gemm(xq, sx, wq, sw, M, N, K, y, ydt, ldy, nullptr, 0, stream);
  if (need > (size_t)SQ_NOALLOC_SCRATCH_BYTES) return SQ_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return SQ_ERR_CUDA;
  return sq_w8a8_gemm(xq, sx, wq, sw, M, N, K, y, ydt, ldy, scratch, (size_t)SQ_NOALLOC_SCRATCH_BYTES, stream);
}

// sq_api.cu -- the C ABI (include/sq_w8a8.h): argument validation on the host, then one
// launch of the matching sm_100a kernel on the caller's stream.  Validation runs before
// any CUDA call, so a bad argument returns its status with nothing enqueued (and without
// touching the device at all).
#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>

#include "sq_common.cuh"

namespace sqh {
cudaError_t launch_absmax(const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, int axis, int accumulate,
                          float* out, cudaStream_t st);
cudaError_t launch_calib_ln_absmax(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ld, const float* gamma,
                                   const float* beta, float eps, int accumulate, float* out, cudaStream_t st);
cudaError_t launch_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s, cudaStream_t st);
cudaError_t launch_fold_quant(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw, const float* s,
                              const float* gamma, const float* beta, int8_t* Wq, float* sw, float* gamma_f,
                              float* beta_f, cudaStream_t st);
cudaError_t launch_ln_smooth_quant(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                                   const float* beta_f, const float* s, float eps, int8_t* xq, float* sx,
                                   cudaStream_t st);
cudaError_t launch_ln_smooth_quant_per_tensor(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx,
                                              const float* gamma_f, const float* beta_f, const float* s, float eps,
                                              int static_scale, float* scale, int8_t* xq, float* sx,
                                              cudaStream_t st);
cudaError_t launch_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M, int64_t N,
                        int64_t K, void* y, int ydt, int64_t ldy, void* ws, size_t ws_bytes, float* rowmax,
                        cudaStream_t st, bool* ws_too_small);
cudaError_t launch_quant_codes(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx, const float* rowmax,
                               int8_t* xq, float* sx, cudaStream_t st);
cudaError_t launch_fold_next_smoothing(const float* sw, const float* s_next, int64_t N, float* out, cudaStream_t st);
cudaError_t launch_fold_quant_fp8(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw, const float* s,
                                  const float* gamma, const float* beta, uint8_t* Wq, float* sw, float* gamma_f,
                                  float* beta_f, cudaStream_t st);
cudaError_t launch_ln_smooth_quant_fp8(const void* x, bool bf16, int64_t M, int64_t K, int64_t ldx,
                                       const float* gamma_f, const float* beta_f, const float* s, float eps,
                                       uint8_t* xq, float* sx, cudaStream_t st);
cudaError_t launch_gemm_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw, int64_t M,
                            int64_t N, int64_t K, void* y, int ydt, int64_t ldy, void* ws, size_t ws_bytes,
                            cudaStream_t st, bool* ws_too_small);
size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K);
int fold_kernel_launches(const void* W, bool bf16, int64_t K, int64_t N, int64_t ldw);
cudaError_t read_device_error(unsigned int* code, int clear, cudaStream_t st);
cudaError_t set_wait_limit(unsigned long long ns, cudaStream_t st);

namespace {
constexpr int kMaxDevices = 64;
int g_sms[kMaxDevices];
std::once_flag g_once[kMaxDevices];
}  // namespace

// Occupancy queries for clusters take long enough to show up in short kernels' launch time;
// the answer depends only on the kernel, the device and the launch shape, so it is kept.
cudaError_t max_active_clusters(const void* kern, const cudaLaunchConfig_t* cfg, int* clusters) {
  static std::mutex mu;
  static std::map<std::tuple<int, const void*, size_t, unsigned, unsigned>, int> cache;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  unsigned cx = 1;
  for (unsigned i = 0; i < cfg->numAttrs; ++i)
    if (cfg->attrs[i].id == cudaLaunchAttributeClusterDimension) cx = cfg->attrs[i].val.clusterDim.x;
  const auto key = std::make_tuple(dev, kern, cfg->dynamicSmemBytes, cfg->blockDim.x, cx);
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find(key);
    if (it != cache.end()) {
      *clusters = it->second;
      return cudaSuccess;
    }
  }
  e = cudaOccupancyMaxActiveClusters(clusters, kern, cfg);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = *clusters;
  return cudaSuccess;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  std::call_once(g_once[dev], [dev] {
    int v = 0;
    g_sms[dev] = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && v > 0 ? v : 148;
  });
  return g_sms[dev];
}

}  // namespace sqh

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
int elt_size(sq_dtype dt) { return dt == SQ_BF16 ? 2 : 4; }
bool input_dtype_ok(sq_dtype dt) { return dt == SQ_BF16 || dt == SQ_F32; }
cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
sq_status cuda_status(cudaError_t e) { return e == cudaSuccess ? SQ_OK : SQ_ERR_CUDA; }

// Checks of a dense row-major input matrix used by the vector-load kernels.
sq_status check_matrix(const void* x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld) {
  if (!input_dtype_ok(dt)) return SQ_ERR_INVALID_ARG;
  if (rows < 0 || cols < 0 || ld < cols) return SQ_ERR_INVALID_ARG;
  if (rows > 0 && cols > 0 && x == nullptr) return SQ_ERR_INVALID_ARG;
  const int e = elt_size(dt);
  if (!aligned16(x) || (cols * e) % 16 != 0 || (ld * e) % 16 != 0) return SQ_ERR_ALIGNMENT;
  return SQ_OK;
}

bool vec_ok(const float* p) { return p != nullptr && aligned16(p); }

}  // namespace

namespace {
// Validation shared by the INT8 and FP8 folds; SQ_OK with *empty set means nothing to do.
sq_status check_fold(const void* W, sq_dtype dt, int64_t K, int64_t N, int64_t ldw, const float* s,
                     const float* gamma, const float* beta, const void* Wq, const float* sw, const float* gamma_f,
                     const float* beta_f, bool* empty) {
  *empty = false;
  if (K < 0 || N < 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_matrix(W, dt, K, N, ldw);
  if (st != SQ_OK) return st;
  if (K == 0 || N == 0) {
    *empty = true;
    return SQ_OK;
  }
  if (s == nullptr || !aligned4(s) || Wq == nullptr || sw == nullptr || !aligned4(sw)) return SQ_ERR_INVALID_ARG;
  if ((gamma && !aligned4(gamma)) || (beta && !aligned4(beta)) || (gamma_f && !aligned4(gamma_f)) ||
      (beta_f && !aligned4(beta_f)))
    return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || !aligned16(Wq)) return SQ_ERR_ALIGNMENT;
  if (K > SQ_MAX_K) return SQ_ERR_UNSUPPORTED;
  return SQ_OK;
}

// Validation shared by the per-token INT8 and FP8 quantisers.
sq_status check_row_quant(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                          const float* beta_f, const float* s, float eps, const void* xq, const float* sx,
                          bool* empty) {
  *empty = false;
  if (M < 0 || K <= 0) return SQ_ERR_INVALID_ARG;
  if ((gamma_f == nullptr) == (s == nullptr)) return SQ_ERR_INVALID_ARG;  // exactly one mode
  if (gamma_f == nullptr && beta_f != nullptr) return SQ_ERR_INVALID_ARG;
  sq_status st = check_matrix(x, dt, M, K, ldx);
  if (st != SQ_OK) return st;
  if ((gamma_f && !aligned16(gamma_f)) || (beta_f && !aligned16(beta_f)) || (s && !aligned16(s)))
    return SQ_ERR_ALIGNMENT;
  if (gamma_f && !(eps >= 0.0f)) return SQ_ERR_INVALID_ARG;
  if (M == 0) {
    *empty = true;
    return SQ_OK;
  }
  if (xq == nullptr || sx == nullptr || !aligned4(sx)) return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || !aligned16(xq)) return SQ_ERR_ALIGNMENT;
  if (K > SQ_MAX_K_ROW || (dt == SQ_F32 && K > SQ_MAX_K_ROW / 2)) return SQ_ERR_UNSUPPORTED;
  if (M > (int64_t)INT32_MAX) return SQ_ERR_UNSUPPORTED;
  return SQ_OK;
}

// Validation shared by the INT8 and FP8 GEMMs (the FP8 one has no int32 output).
sq_status check_gemm(const void* xq, const float* sx, const void* wq, const float* sw, int64_t M, int64_t N,
                     int64_t K, const void* y, sq_dtype ydt, int64_t ldy, const void* workspace, bool allow_i32,
                     bool* empty) {
  *empty = false;
  if (M < 0 || N < 0 || K <= 0) return SQ_ERR_INVALID_ARG;
  if (ydt != SQ_BF16 && ydt != SQ_F32 && !(allow_i32 && ydt == SQ_I32)) return SQ_ERR_INVALID_ARG;
  if (ldy < N) return SQ_ERR_INVALID_ARG;
  if (M == 0 || N == 0) {
    *empty = true;
    return SQ_OK;
  }
  if (!xq || !wq || !y) return SQ_ERR_INVALID_ARG;
  if (ydt != SQ_I32 && (!sx || !sw || !aligned4(sx) || !aligned4(sw))) return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || !aligned16(xq) || !aligned16(wq)) return SQ_ERR_ALIGNMENT;
  const uintptr_t e = ydt == SQ_BF16 ? 2 : 4;
  if (reinterpret_cast<uintptr_t>(y) % e != 0) return SQ_ERR_ALIGNMENT;
  if (workspace && (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SQ_ERR_ALIGNMENT;
  if (K > SQ_MAX_K) return SQ_ERR_UNSUPPORTED;
  if (M > (int64_t)INT32_MAX || N > (int64_t)INT32_MAX) return SQ_ERR_UNSUPPORTED;
  return SQ_OK;
}
}  // namespace

namespace sqh {
// The argument checks of sq_w8a8_gemm (for entry points that wrap it); *empty is set when the
// shape is empty and nothing is to be launched.
sq_status check_gemm_args(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M, int64_t N,
                          int64_t K, const void* y, sq_dtype ydt, int64_t ldy, bool* empty) {
  return check_gemm(xq, sx, wq, sw, M, N, K, y, ydt, ldy, nullptr, true, empty);
}
}  // namespace sqh

extern "C" {

int sq_abi_version(void) { return 102; }

const char* sq_status_string(sq_status status) {
  switch (status) {
    case SQ_OK: return "SQ_OK";
    case SQ_ERR_INVALID_ARG: return "SQ_ERR_INVALID_ARG";
    case SQ_ERR_UNSUPPORTED: return "SQ_ERR_UNSUPPORTED";
    case SQ_ERR_ALIGNMENT: return "SQ_ERR_ALIGNMENT";
    case SQ_ERR_CUDA: return "SQ_ERR_CUDA";
    case SQ_ERR_WORKSPACE: return "SQ_ERR_WORKSPACE";
  }
  return "SQ_ERR_UNKNOWN";
}

sq_status sq_calib_absmax(const void* x, sq_dtype dt, int64_t rows, int64_t cols, int64_t ld, int axis,
                          int accumulate, float* out, void* stream) {
  if (axis != 0 && axis != 1) return SQ_ERR_INVALID_ARG;
  if (accumulate != 0 && accumulate != 1) return SQ_ERR_INVALID_ARG;
  sq_status st = check_matrix(x, dt, rows, cols, ld);
  if (st != SQ_OK) return st;
  const int64_t nout = axis == 0 ? cols : rows;
  if (nout > 0 && (out == nullptr || !aligned4(out))) return SQ_ERR_INVALID_ARG;
  if (rows > (int64_t)INT32_MAX) return SQ_ERR_UNSUPPORTED;
  if (nout == 0) return SQ_OK;
  if (rows == 0 || cols == 0) {
    // an empty reduction: max over nothing is 0 (the identity for absolute values)
    if (accumulate) return SQ_OK;
    return cuda_status(cudaMemsetAsync(out, 0, sizeof(float) * (size_t)nout, as_stream(stream)));
  }
  return cuda_status(sqh::launch_absmax(x, dt == SQ_BF16, rows, cols, ld, axis, accumulate, out, as_stream(stream)));
}

sq_status sq_calib_ln_absmax(const void* x, sq_dtype dt, int64_t rows, int64_t K, int64_t ldx, const float* gamma,
                             const float* beta, float eps, int accumulate, float* out, void* stream) {
  if (accumulate != 0 && accumulate != 1) return SQ_ERR_INVALID_ARG;
  if (K <= 0 || rows < 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_matrix(x, dt, rows, K, ldx);
  if (st != SQ_OK) return st;
  if (!vec_ok(gamma) || (beta && !aligned16(beta)) || out == nullptr || !aligned4(out)) return SQ_ERR_INVALID_ARG;
  if (!(eps >= 0.0f)) return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0) return SQ_ERR_ALIGNMENT;
  if (K > SQ_MAX_K_ROW || (dt == SQ_F32 && K > SQ_MAX_K_ROW / 2)) return SQ_ERR_UNSUPPORTED;
  if (rows == 0) {
    if (accumulate) return SQ_OK;
    return cuda_status(cudaMemsetAsync(out, 0, sizeof(float) * (size_t)K, as_stream(stream)));
  }
  return cuda_status(
      sqh::launch_calib_ln_absmax(x, dt == SQ_BF16, rows, K, ldx, gamma, beta, eps, accumulate, out, as_stream(stream)));
}

sq_status sq_smooth_factors(const float* ax, const float* aw, int64_t K, float alpha, float* s, void* stream) {
  if (K < 0) return SQ_ERR_INVALID_ARG;
  if (!(alpha >= 0.0f && alpha <= 1.0f)) return SQ_ERR_INVALID_ARG;
  if (K == 0) return SQ_OK;
  if (!ax || !aw || !s || !aligned4(ax) || !aligned4(aw) || !aligned4(s)) return SQ_ERR_INVALID_ARG;
  return cuda_status(sqh::launch_smooth_factors(ax, aw, K, alpha, s, as_stream(stream)));
}

sq_status sq_fold_next_smoothing(const float* sw, const float* s_next, int64_t N, float* sw_out, void* stream) {
  if (N < 0) return SQ_ERR_INVALID_ARG;
  if (N == 0) return SQ_OK;
  if (!sw || !s_next || !sw_out || !aligned4(sw) || !aligned4(s_next) || !aligned4(sw_out)) return SQ_ERR_INVALID_ARG;
  return cuda_status(sqh::launch_fold_next_smoothing(sw, s_next, N, sw_out, as_stream(stream)));
}

sq_status sq_fold_quant_weights_fp8(const void* W, sq_dtype dt, int64_t K, int64_t N, int64_t ldw, const float* s,
                                    const float* gamma, const float* beta, uint8_t* Wq, float* sw, float* gamma_f,
                                    float* beta_f, void* stream) {
  bool empty = false;
  const sq_status st = check_fold(W, dt, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, &empty);
  if (st != SQ_OK || empty) return st;
  return cuda_status(sqh::launch_fold_quant_fp8(W, dt == SQ_BF16, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f,
                                                as_stream(stream)));
}

sq_status sq_ln_smooth_quant_fp8(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                                 const float* beta_f, const float* s, float eps, uint8_t* xq, float* sx,
                                 void* stream) {
  bool empty = false;
  const sq_status st = check_row_quant(x, dt, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, &empty);
  if (st != SQ_OK || empty) return st;
  return cuda_status(sqh::launch_ln_smooth_quant_fp8(x, dt == SQ_BF16, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx,
                                                     as_stream(stream)));
}

sq_status sq_w8a8_gemm_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw, int64_t M,
                           int64_t N, int64_t K, void* y, sq_dtype ydt, int64_t ldy, void* workspace,
                           size_t ws_bytes, void* stream) {
  bool empty = false;
  const sq_status st = check_gemm(xq, sx, wq, sw, M, N, K, y, ydt, ldy, workspace, false, &empty);
  if (st != SQ_OK || empty) return st;
  bool ws_small = false;
  cudaError_t err = sqh::launch_gemm_fp8(xq, sx, wq, sw, M, N, K, y, (int)ydt, ldy, workspace, ws_bytes,
                                         as_stream(stream), &ws_small);
  if (ws_small) return SQ_ERR_WORKSPACE;
  return cuda_status(err);
}

sq_status sq_fold_quant_weights(const void* W, sq_dtype dt, int64_t K, int64_t N, int64_t ldw, const float* s,
                                const float* gamma, const float* beta, int8_t* Wq, float* sw, float* gamma_f,
                                float* beta_f, void* stream) {
  bool empty = false;
  const sq_status st = check_fold(W, dt, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f, &empty);
  if (st != SQ_OK || empty) return st;
  return cuda_status(sqh::launch_fold_quant(W, dt == SQ_BF16, K, N, ldw, s, gamma, beta, Wq, sw, gamma_f, beta_f,
                                            as_stream(stream)));
}

int sq_fold_kernel_launches(const void* W, sq_dtype dt, int64_t K, int64_t N, int64_t ldw) {
  return sqh::fold_kernel_launches(W, dt == SQ_BF16, K, N, ldw);
}

sq_status sq_ln_smooth_quant(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx, const float* gamma_f,
                             const float* beta_f, const float* s, float eps, int8_t* xq, float* sx, void* stream) {
  bool empty = false;
  const sq_status st = check_row_quant(x, dt, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, &empty);
  if (st != SQ_OK || empty) return st;
  return cuda_status(
      sqh::launch_ln_smooth_quant(x, dt == SQ_BF16, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, as_stream(stream)));
}

sq_status sq_ln_smooth_quant_per_tensor(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx,
                                        const float* gamma_f, const float* beta_f, const float* s, float eps,
                                        int static_scale, float* scale, int8_t* xq, float* sx, void* stream) {
  if (static_scale != 0 && static_scale != 1) return SQ_ERR_INVALID_ARG;
  if (scale == nullptr || !aligned4(scale)) return SQ_ERR_INVALID_ARG;
  bool empty = false;
  const sq_status st = check_row_quant(x, dt, M, K, ldx, gamma_f, beta_f, s, eps, xq, sx, &empty);
  if (st != SQ_OK || empty) return st;
  return cuda_status(sqh::launch_ln_smooth_quant_per_tensor(x, dt == SQ_BF16, M, K, ldx, gamma_f, beta_f, s, eps,
                                                            static_scale, scale, xq, sx, as_stream(stream)));
}

size_t sq_w8a8_gemm_workspace_size(int64_t M, int64_t N, int64_t K) {
  if (M < 0 || N < 0 || K <= 0 || K > SQ_MAX_K || K % 16 != 0) return (size_t)-1;
  if (M == 0 || N == 0) return 0;
  return sqh::gemm_workspace_size(M, N, K);
}

sq_status sq_w8a8_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M, int64_t N,
                       int64_t K, void* y, sq_dtype ydt, int64_t ldy, void* workspace, size_t ws_bytes, void* stream) {
  bool empty = false;
  const sq_status st = check_gemm(xq, sx, wq, sw, M, N, K, y, ydt, ldy, workspace, true, &empty);
  if (st != SQ_OK || empty) return st;
  bool ws_small = false;
  cudaError_t err = sqh::launch_gemm(xq, sx, wq, sw, M, N, K, y, (int)ydt, ldy, workspace, ws_bytes, nullptr,
                                     as_stream(stream), &ws_small);
  if (ws_small) return SQ_ERR_WORKSPACE;
  return cuda_status(err);
}

sq_status sq_w8a8_gemm_rowmax(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M,
                              int64_t N, int64_t K, void* y, sq_dtype ydt, int64_t ldy, float* rowmax, void* workspace,
                              size_t ws_bytes, void* stream) {
  if (ydt != SQ_BF16 && ydt != SQ_F32) return SQ_ERR_INVALID_ARG;
  bool empty = false;
  const sq_status st = check_gemm(xq, sx, wq, sw, M, N, K, y, ydt, ldy, workspace, false, &empty);
  if (st != SQ_OK || empty) return st;
  if (rowmax == nullptr || !aligned4(rowmax)) return SQ_ERR_INVALID_ARG;
  bool ws_small = false;
  cudaError_t err = sqh::launch_gemm(xq, sx, wq, sw, M, N, K, y, (int)ydt, ldy, workspace, ws_bytes, rowmax,
                                     as_stream(stream), &ws_small);
  if (ws_small) return SQ_ERR_WORKSPACE;
  return cuda_status(err);
}

sq_status sq_quant_codes(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx, const float* rowmax, int8_t* xq,
                         float* sx, void* stream) {
  if (M < 0 || K <= 0) return SQ_ERR_INVALID_ARG;
  sq_status st = check_matrix(x, dt, M, K, ldx);
  if (st != SQ_OK) return st;
  if (M == 0) return SQ_OK;
  if (rowmax == nullptr || !aligned4(rowmax) || xq == nullptr || sx == nullptr || !aligned4(sx))
    return SQ_ERR_INVALID_ARG;
  if (K % 16 != 0 || !aligned16(xq)) return SQ_ERR_ALIGNMENT;
  if (M > (int64_t)INT32_MAX) return SQ_ERR_UNSUPPORTED;
  return cuda_status(sqh::launch_quant_codes(x, dt == SQ_BF16, M, K, ldx, rowmax, xq, sx, as_stream(stream)));
}

sq_status sq_set_wait_limit(unsigned long long ns, void* stream) {
  return cuda_status(sqh::set_wait_limit(ns, as_stream(stream)));
}

sq_status sq_device_error(unsigned int* code, int clear, void* stream) {
  if (code == nullptr) return SQ_ERR_INVALID_ARG;
  return cuda_status(sqh::read_device_error(code, clear, as_stream(stream)));
}

}  // extern "C"

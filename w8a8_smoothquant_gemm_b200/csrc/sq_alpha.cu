// sq_alpha.cu -- migration strength by grid search on calibration data.
//
// "4.2 W8A8 量化与 SmoothQuant", sec. 5.2: alpha is fixed once, offline, by a grid search over
// calibration samples.  "量化：只压权重，与训练后量化（PTQ）", AWQ paragraph: the data-only form
// of that search minimises the layer-output error || Q(W diag(s)) (diag(s)^-1 X) - W X || over
// a grid of alpha in [0, 1].  For every candidate the whole W8A8 layer of this library runs
// on the calibration batch:
//   s = s(ax, aw, alpha) -> fold + per-channel weight codes -> (LayerNorm +) smooth +
//   per-token codes -> INT8 GEMM with the binary32 epilogue ((float)acc * sx) * sw = Y_hat,
// and err = ||Y_hat - Y||_F^2 / ||Y||_F^2 against the reference Y = X_in W, where X_in is the
// layer's input (LN(x; gamma, beta) with the fixed-order statistics, or x) and the reference
// product accumulates binary32 products in a fixed k order on the CUDA cores (it is the
// yardstick, not the hot path, and wants full binary32 inputs).
#include <algorithm>

#include "sq_rowln.cuh"

namespace sqk {

// X_in = LN(x; gamma, beta) as binary32 rows (one block of 256 threads per row; the same
// statistics and apply as the quantiser kernels, so X_in is the quantiser's y with the
// unfolded gamma, beta).
template <bool BF16, int MAXC>
__global__ void __launch_bounds__(ROW_THREADS)
layernorm_rows_kernel(const char* __restrict__ x, int64_t M, int K, int64_t ld_bytes, const float* __restrict__ gamma,
                      const float* __restrict__ beta, float eps, float* __restrict__ out) {
  __shared__ float red[2 * (ROW_WARPS + 1)];
  const int nchunks = K / 8;
  for (int64_t m = blockIdx.x; m < M; m += gridDim.x) {
    RowChunks<BF16, MAXC> rc;
    rc.load(x + m * ld_bytes, nchunks);
    float mu, rstd;
    row_stats(rc, nchunks, K, eps, red, mu, rstd);
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = threadIdx.x + i * ROW_THREADS;
      if (c < nchunks) {
        float f[8], y[8];
        rc.get(i, f);
        ln_chunk(f, mu, rstd, gamma, beta, c, y);
        float4* o = reinterpret_cast<float4*>(out + m * (int64_t)K + (int64_t)c * 8);
        o[0] = make_float4(y[0], y[1], y[2], y[3]);
        o[1] = make_float4(y[4], y[5], y[6], y[7]);
      }
    }
    __syncthreads();  // `red` is reused by the next row
  }
}

template <bool BF16>
__device__ __forceinline__ float load_elt(const void* p, int64_t i) {
  if (BF16) return __uint_as_float((uint32_t)reinterpret_cast<const uint16_t*>(p)[i] << 16);
  return reinterpret_cast<const float*>(p)[i];
}

// Reference product Y[M, N] = A[M, K] W[K, N] in binary32, k in increasing order per output
// (fused multiply-add, one rounding per step).  128 x 128 output tiles, 8-deep k slabs in
// double-buffered shared memory, 8 x 8 outputs per thread as packed binary32 pairs (each
// half rounds as the scalar fma would).
template <bool ABF16, bool WBF16>
__global__ void __launch_bounds__(256, 2)
reference_gemm_kernel(const void* __restrict__ A, int64_t lda, const void* __restrict__ W, int64_t ldw, int64_t M,
                      int64_t N, int64_t K, float* __restrict__ Y) {
  __shared__ __align__(16) float As[2][8][128];  // [k][m]
  __shared__ __align__(16) float Ws[2][8][128];  // [k][n]
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int64_t m0 = (int64_t)blockIdx.y * 128, n0 = (int64_t)blockIdx.x * 128;
  // staging assignment: A tile 128 rows x 8 k (thread: row ar, k ak..ak+3), W tile 8 k x 128
  // columns (thread: k wk, columns wc..wc+3)
  const int ar = threadIdx.x / 2, ak = (threadIdx.x % 2) * 4;
  const int wk = threadIdx.x / 32, wc = (threadIdx.x % 32) * 4;
  float ra[4], rw[4];
  // K % 8 == 0, and rows start on 16-byte boundaries: 4 consecutive elements load as one
  // 8-byte (bf16) or 16-byte (fp32) vector
  auto load4 = [](const void* base, int64_t i, bool bf16, float* out) {
    if (bf16) {
      const uint2 u = __ldg(reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(base) + i));
      out[0] = bf16lo(u.x); out[1] = bf16hi(u.x); out[2] = bf16lo(u.y); out[3] = bf16hi(u.y);
    } else {
      const float4 f = __ldg(reinterpret_cast<const float4*>(reinterpret_cast<const float*>(base) + i));
      out[0] = f.x; out[1] = f.y; out[2] = f.z; out[3] = f.w;
    }
  };
  auto fetch = [&](int64_t k0) {
    const int64_t m = m0 + ar;
    if (m < M) load4(A, m * lda + k0 + ak, ABF16, ra);
    else ra[0] = ra[1] = ra[2] = ra[3] = 0.0f;
    const int64_t k2 = k0 + wk, n = n0 + wc;
    if (n + 3 < N) {
      load4(W, k2 * ldw + n, WBF16, rw);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) rw[i] = (n + i < N) ? load_elt<WBF16>(W, k2 * ldw + n + i) : 0.0f;
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int i = 0; i < 4; ++i) As[buf][ak + i][ar] = ra[i];
    *reinterpret_cast<float4*>(&Ws[buf][wk][wc]) = make_float4(rw[0], rw[1], rw[2], rw[3]);
  };
  float2 acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = make_float2(0.0f, 0.0f);
  fetch(0);
  stash(0);
  __syncthreads();
  int buf = 0;
  for (int64_t k0 = 0; k0 < K; k0 += 8) {
    const bool more = k0 + 8 < K;
    if (more) fetch(k0 + 8);  // next slab into registers while this one is used
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 8 + 4]);
      const float4 w0 = *reinterpret_cast<const float4*>(&Ws[buf][kk][tx * 8]);
      const float4 w1 = *reinterpret_cast<const float4*>(&Ws[buf][kk][tx * 8 + 4]);
      const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float2 w[4] = {make_float2(w0.x, w0.y), make_float2(w0.z, w0.w), make_float2(w1.x, w1.y),
                           make_float2(w1.z, w1.w)};
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = __ffma2_rn(make_float2(a[i], a[i]), w[j], acc[i][j]);
    }
    if (more) {
      stash(buf ^ 1);
      __syncthreads();
      buf ^= 1;
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int64_t m = m0 + ty * 8 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t n = n0 + tx * 8 + 2 * j;
      if (n < N) Y[m * N + n] = acc[i][j].x;
      if (n + 1 < N) Y[m * N + n + 1] = acc[i][j].y;
    }
  }
}

// acc[0] += sum (Yh - Y)^2, or (Yh == NULL) sum Y^2, in binary64.
__global__ void __launch_bounds__(256)
sq_error_kernel(const float* __restrict__ Yh, const float* __restrict__ Y, int64_t n, double* __restrict__ acc) {
  __shared__ double red[8];
  double s = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * 256 + threadIdx.x; i < n; i += (int64_t)gridDim.x * 256) {
    const double d = Yh ? (double)Yh[i] - (double)Y[i] : (double)Y[i];
    s += d * d;
  }
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < 8; ++w) t += red[w];
    atomicAdd(acc, t);
  }
}

// err[i] = num[i] / den (den = num[n]).
__global__ void finish_kernel(const double* __restrict__ num, int n, double* __restrict__ err) {
  const int i = threadIdx.x;
  if (i < n) err[i] = num[n] > 0.0 ? num[i] / num[n] : 0.0;
}

}  // namespace sqk

namespace {

constexpr int kMaxAlphas = 256;

size_t align256(size_t b) { return (b + 255) & ~size_t(255); }

// Workspace slices of the search (each 256-byte aligned).
struct AlphaWs {
  float *ax, *aw, *s, *gf, *bf, *sw, *sx, *xin, *y, *yh;
  int8_t *wq, *xq;
  double* acc;
  void* gemm_ws;
  size_t gemm_ws_bytes, total;
};

AlphaWs carve(void* base, int64_t M, int64_t K, int64_t N, bool ln) {
  AlphaWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {  // (base may be NULL when only the total is wanted)
    char* p = reinterpret_cast<char*>(reinterpret_cast<uintptr_t>(base) + off);
    off += align256(bytes);
    return p;
  };
  w.ax = reinterpret_cast<float*>(take(4 * K));
  w.aw = reinterpret_cast<float*>(take(4 * K));
  w.s = reinterpret_cast<float*>(take(4 * K));
  w.gf = reinterpret_cast<float*>(take(4 * K));
  w.bf = reinterpret_cast<float*>(take(4 * K));
  w.sw = reinterpret_cast<float*>(take(4 * N));
  w.sx = reinterpret_cast<float*>(take(4 * M));
  w.wq = reinterpret_cast<int8_t*>(take((size_t)N * K));
  w.xq = reinterpret_cast<int8_t*>(take((size_t)M * K));
  w.xin = ln ? reinterpret_cast<float*>(take(4 * (size_t)M * K)) : nullptr;
  w.y = reinterpret_cast<float*>(take(4 * (size_t)M * N));
  w.yh = reinterpret_cast<float*>(take(4 * (size_t)M * N));
  w.acc = reinterpret_cast<double*>(take(8 * (kMaxAlphas + 1)));
  w.gemm_ws_bytes = sq_w8a8_gemm_workspace_size(M, N, K);
  w.gemm_ws = w.gemm_ws_bytes ? take(w.gemm_ws_bytes) : nullptr;
  w.total = off;
  return w;
}

template <bool BF16>
cudaError_t launch_layernorm_rows(const void* x, int64_t M, int64_t K, int64_t ldx, const float* gamma,
                                  const float* beta, float eps, float* out, cudaStream_t st) {
  const int need = (int)((K / 8 + sqk::ROW_THREADS - 1) / sqk::ROW_THREADS);
  const int64_t ldb = ldx * (BF16 ? 2 : 4);
  const unsigned grid = (unsigned)std::min<int64_t>(M, 148 * 8);
  const int k = (int)K;
#define SQ_LN_ROWS(C)                                                                                        \
  if (need <= C) {                                                                                           \
    sqk::layernorm_rows_kernel<BF16, C><<<grid, sqk::ROW_THREADS, 0, st>>>((const char*)x, M, k, ldb, gamma, \
                                                                          beta, eps, out);                   \
    return cudaGetLastError();                                                                               \
  }
  SQ_LN_ROWS(1) SQ_LN_ROWS(2) SQ_LN_ROWS(4) SQ_LN_ROWS(8) SQ_LN_ROWS(16)
  if (BF16) SQ_LN_ROWS(32)
#undef SQ_LN_ROWS
  return cudaErrorInvalidValue;
}

cudaError_t launch_reference_gemm(const void* A, bool abf16, int64_t lda, const void* W, bool wbf16, int64_t ldw,
                                  int64_t M, int64_t N, int64_t K, float* Y, cudaStream_t st) {
  const dim3 grid((unsigned)((N + 127) / 128), (unsigned)((M + 127) / 128));
  if (abf16 && wbf16) sqk::reference_gemm_kernel<true, true><<<grid, 256, 0, st>>>(A, lda, W, ldw, M, N, K, Y);
  else if (abf16) sqk::reference_gemm_kernel<true, false><<<grid, 256, 0, st>>>(A, lda, W, ldw, M, N, K, Y);
  else if (wbf16) sqk::reference_gemm_kernel<false, true><<<grid, 256, 0, st>>>(A, lda, W, ldw, M, N, K, Y);
  else sqk::reference_gemm_kernel<false, false><<<grid, 256, 0, st>>>(A, lda, W, ldw, M, N, K, Y);
  return cudaGetLastError();
}

cudaError_t launch_sq_error(const float* yh, const float* y, int64_t n, double* acc, cudaStream_t st) {
  const unsigned grid = (unsigned)std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 8));
  sqk::sq_error_kernel<<<grid, 256, 0, st>>>(yh, y, n, acc);
  return cudaGetLastError();
}

#define SQ_TRY(call)                        \
  do {                                      \
    const sq_status st_ = (call);           \
    if (st_ != SQ_OK) return st_;           \
  } while (0)
#define SQ_TRY_CUDA(call)                     \
  do {                                        \
    if ((call) != cudaSuccess) return SQ_ERR_CUDA; \
  } while (0)

}  // namespace

extern "C" {

size_t sq_alpha_search_workspace_size(int64_t M, int64_t K, int64_t N) {
  if (M <= 0 || N <= 0 || K <= 0 || K % 16 != 0 || K > SQ_MAX_K_ROW) return (size_t)-1;
  return carve(nullptr, M, K, N, true).total;
}

sq_status sq_alpha_search(const void* x, sq_dtype dt, int64_t M, int64_t K, int64_t ldx, const float* gamma,
                          const float* beta, float eps, const void* W, sq_dtype wdt, int64_t N, int64_t ldw,
                          const float* alphas, int n_alpha, double* err, void* workspace, size_t ws_bytes,
                          void* stream) {
  if (M <= 0 || N <= 0 || K <= 0) return SQ_ERR_INVALID_ARG;
  if (alphas == nullptr || n_alpha < 1 || n_alpha > kMaxAlphas || err == nullptr) return SQ_ERR_INVALID_ARG;
  for (int i = 0; i < n_alpha; ++i)
    if (!(alphas[i] >= 0.0f && alphas[i] <= 1.0f)) return SQ_ERR_INVALID_ARG;
  if (gamma == nullptr && beta != nullptr) return SQ_ERR_INVALID_ARG;
  if ((dt != SQ_BF16 && dt != SQ_F32) || (wdt != SQ_BF16 && wdt != SQ_F32)) return SQ_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(err) % 8 != 0) return SQ_ERR_ALIGNMENT;
  if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return SQ_ERR_ALIGNMENT;
  const size_t need = sq_alpha_search_workspace_size(M, K, N);
  if (need == (size_t)-1) return K % 16 != 0 ? SQ_ERR_ALIGNMENT : SQ_ERR_UNSUPPORTED;
  if (ws_bytes < need) return SQ_ERR_WORKSPACE;
  const bool ln = gamma != nullptr;
  const AlphaWs w = carve(workspace, M, K, N, ln);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // the GEMM's workspace starts zeroed (its tile sums); the caller's buffer may hold anything
  if (w.gemm_ws) SQ_TRY_CUDA(cudaMemsetAsync(w.gemm_ws, 0, w.gemm_ws_bytes, st));

  // statistics of the layer input and the weights (the checks of these calls cover x and W)
  if (ln) SQ_TRY(sq_calib_ln_absmax(x, dt, M, K, ldx, gamma, beta, eps, 0, w.ax, stream));
  else SQ_TRY(sq_calib_absmax(x, dt, M, K, ldx, 0, 0, w.ax, stream));
  SQ_TRY(sq_calib_absmax(W, wdt, K, N, ldw, 1, 0, w.aw, stream));
  // reference Y = X_in W and its squared norm
  if (ln) {
    SQ_TRY_CUDA(dt == SQ_BF16 ? launch_layernorm_rows<true>(x, M, K, ldx, gamma, beta, eps, w.xin, st)
                              : launch_layernorm_rows<false>(x, M, K, ldx, gamma, beta, eps, w.xin, st));
    SQ_TRY_CUDA(launch_reference_gemm(w.xin, false, K, W, wdt == SQ_BF16, ldw, M, N, K, w.y, st));
  } else {
    SQ_TRY_CUDA(launch_reference_gemm(x, dt == SQ_BF16, ldx, W, wdt == SQ_BF16, ldw, M, N, K, w.y, st));
  }
  SQ_TRY_CUDA(cudaMemsetAsync(w.acc, 0, 8 * (size_t)(n_alpha + 1), st));
  SQ_TRY_CUDA(launch_sq_error(nullptr, w.y, M * N, w.acc + n_alpha, st));
  // the layer at every candidate strength
  for (int i = 0; i < n_alpha; ++i) {
    SQ_TRY(sq_smooth_factors(w.ax, w.aw, K, alphas[i], w.s, stream));
    SQ_TRY(sq_fold_quant_weights(W, wdt, K, N, ldw, w.s, gamma, beta, w.wq, w.sw, ln ? w.gf : nullptr,
                                 ln && beta ? w.bf : nullptr, stream));
    if (ln)
      SQ_TRY(sq_ln_smooth_quant(x, dt, M, K, ldx, w.gf, beta ? w.bf : nullptr, nullptr, eps, w.xq, w.sx, stream));
    else
      SQ_TRY(sq_ln_smooth_quant(x, dt, M, K, ldx, nullptr, nullptr, w.s, eps, w.xq, w.sx, stream));
    SQ_TRY(sq_w8a8_gemm(w.xq, w.sx, w.wq, w.sw, M, N, K, w.yh, SQ_F32, N, w.gemm_ws, w.gemm_ws_bytes, stream));
    SQ_TRY_CUDA(launch_sq_error(w.yh, w.y, M * N, w.acc + i, st));
  }
  sqk::finish_kernel<<<1, kMaxAlphas, 0, st>>>(w.acc, n_alpha, err);
  return cudaGetLastError() == cudaSuccess ? SQ_OK : SQ_ERR_CUDA;
}

}  // extern "C"

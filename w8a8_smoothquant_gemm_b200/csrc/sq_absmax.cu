// sq_absmax.cu -- calibration statistics of SmoothQuant ("4.2 W8A8 量化与 SmoothQuant",
// sec. 4 and 7.1; "量化：只压权重，与训练后量化（PTQ）", SmoothQuant section):
//   per-input-channel activation absmax  max_i |X_ij|      (column max, axis 0)
//   per-input-channel weight absmax       max_k |W_jk|      (row max of W[K, N], axis 1)
//   per-channel absmax of a LayerNorm output, computed without writing it.
//
// All three are HBM-bound single passes: 16-byte vector loads that bypass L1, a
// per-thread running max, a block reduction, and one atomicMax per column per block on
// the float bit pattern (monotone for non-negative floats, so the result is exact and
// independent of order).
#include "sq_ptx.cuh"
#include "sq_rowln.cuh"

namespace sqk {

// ---------------------------------------------------------------------------- axis 0
// Block = 32 column vectors (x) x 8 row lanes (y).  A warp reads 32 consecutive
// 16-byte vectors of one row (512 contiguous bytes).  Each thread walks rows
// r = blockIdx.y * 8 + threadIdx.y + k * gridDim.y * 8, four loads in flight.
constexpr int COL_VX = 32, COL_RY = 8, COL_UNROLL = 4;

template <bool BF16>
__global__ void __launch_bounds__(COL_VX * COL_RY)
absmax_cols_kernel(const char* __restrict__ x, int64_t rows, int64_t nvec, int64_t ld_bytes,
                   float* __restrict__ out) {
  constexpr int EPV = BF16 ? 8 : 4;  // elements per 16-byte vector
  __shared__ float red[COL_RY][COL_VX * EPV + 1];
  const int64_t vec = (int64_t)blockIdx.x * COL_VX + threadIdx.x;
  float m[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) m[e] = 0.0f;
  if (vec < nvec) {
    const int64_t rstep = (int64_t)gridDim.y * COL_RY;
    int64_t r = (int64_t)blockIdx.y * COL_RY + threadIdx.y;
    const char* p = x + vec * 16;
    for (; r + (COL_UNROLL - 1) * rstep < rows; r += COL_UNROLL * rstep) {
      uint4 v[COL_UNROLL];
#pragma unroll
      for (int u = 0; u < COL_UNROLL; ++u) v[u] = ldg_stream16(p + (r + u * rstep) * ld_bytes);
#pragma unroll
      for (int u = 0; u < COL_UNROLL; ++u) {
        if (BF16) {
          float f[8];
          unpack8_bf16(v[u], f);
#pragma unroll
          for (int e = 0; e < EPV; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
        } else {
          const float f[4] = {__uint_as_float(v[u].x), __uint_as_float(v[u].y), __uint_as_float(v[u].z),
                              __uint_as_float(v[u].w)};
#pragma unroll
          for (int e = 0; e < EPV; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
        }
      }
    }
    for (; r < rows; r += rstep) {
      const uint4 v = ldg_stream16(p + r * ld_bytes);
      if (BF16) {
        float f[8];
        unpack8_bf16(v, f);
#pragma unroll
        for (int e = 0; e < EPV; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
      } else {
        const float f[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z), __uint_as_float(v.w)};
#pragma unroll
        for (int e = 0; e < EPV; ++e) m[e] = fmaxf(m[e], fabsf(f[e]));
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPV; ++e) red[threadIdx.y][threadIdx.x * EPV + e] = m[e];
  __syncthreads();
  // 256 threads finish the COL_VX * EPV columns of this block.
  const int tid = threadIdx.y * COL_VX + threadIdx.x;
  for (int c = tid; c < COL_VX * EPV; c += COL_VX * COL_RY) {
    float v = red[0][c];
#pragma unroll
    for (int y = 1; y < COL_RY; ++y) v = fmaxf(v, red[y][c]);
    const int64_t col = (int64_t)blockIdx.x * COL_VX * EPV + c;
    if (col < nvec * EPV) atomic_max_nonneg(out + col, v);
  }
}

// ---------------------------------------------------------------------------- axis 1
// One block of 256 threads per row; the row is read as 16-byte vectors.
template <bool BF16>
__global__ void __launch_bounds__(256)
absmax_rows_kernel(const char* __restrict__ x, int64_t rows, int64_t nvec, int64_t ld_bytes,
                   int accumulate, float* __restrict__ out) {
  __shared__ float red[ROW_WARPS + 1];
  const int64_t r = blockIdx.x;
  const char* p = x + r * ld_bytes;
  float m = 0.0f;
  int64_t v = threadIdx.x;
  for (; v + 3 * 256 < nvec; v += 4 * 256) {
    uint4 q[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) q[u] = ldg_stream16(p + (v + u * 256) * 16);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      if (BF16) {
        float f[8];
        unpack8_bf16(q[u], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
      } else {
        m = fmaxf(fmaxf(m, fabsf(__uint_as_float(q[u].x))), fabsf(__uint_as_float(q[u].y)));
        m = fmaxf(fmaxf(m, fabsf(__uint_as_float(q[u].z))), fabsf(__uint_as_float(q[u].w)));
      }
    }
  }
  for (; v < nvec; v += 256) {
    const uint4 q = ldg_stream16(p + v * 16);
    if (BF16) {
      float f[8];
      unpack8_bf16(q, f);
#pragma unroll
      for (int e = 0; e < 8; ++e) m = fmaxf(m, fabsf(f[e]));
    } else {
      m = fmaxf(fmaxf(m, fabsf(__uint_as_float(q.x))), fabsf(__uint_as_float(q.y)));
      m = fmaxf(fmaxf(m, fabsf(__uint_as_float(q.z))), fabsf(__uint_as_float(q.w)));
    }
  }
  m = block_max(m, red);
  if (threadIdx.x == 0) out[r] = accumulate ? fmaxf(out[r], m) : m;
}

// Short rows (up to 8 KB): one warp per row, every 16-byte vector of the row loaded at once
// (up to 16 per lane in flight), shuffle reduction, no block barrier.
template <bool BF16, int VPL>
__global__ void __launch_bounds__(256)
absmax_rows_warp_kernel(const char* __restrict__ x, int64_t rows, int64_t nvec, int64_t ld_bytes, int accumulate,
                        float* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const char* p = x + r * ld_bytes;
  uint4 q[VPL];
#pragma unroll
  for (int i = 0; i < VPL; ++i)
    if (lane + 32 * i < nvec) q[i] = ldg_stream16(p + (int64_t)(lane + 32 * i) * 16);
  float m[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    if (lane + 32 * i < nvec) {
      if (BF16) {
        float f[8];
        unpack8_bf16(q[i], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) m[e & 3] = fmaxf(m[e & 3], fabsf(f[e]));
      } else {
        m[0] = fmaxf(m[0], fabsf(__uint_as_float(q[i].x)));
        m[1] = fmaxf(m[1], fabsf(__uint_as_float(q[i].y)));
        m[2] = fmaxf(m[2], fabsf(__uint_as_float(q[i].z)));
        m[3] = fmaxf(m[3], fabsf(__uint_as_float(q[i].w)));
      }
    }
  }
  float v = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  if (lane == 0) out[r] = accumulate ? fmaxf(out[r], v) : v;
}

// ---------------------------------------------------------------------------- LayerNorm output
// Blocks loop over rows; each thread keeps the running max of the elements of its own
// chunks -- in registers (REG, rows of up to 32 elements per thread) or in shared memory --
// then one atomicMax per column per block.  With rows_atomic set (K too large for shared
// memory) the running max goes straight to global memory with an atomic per element per row.
// Launched in clusters (shared-memory maxima only), the blocks of a cluster first combine
// their maxima through distributed shared memory and each column takes one atomicMax per
// cluster: with a few rows per block (2048 rows of 12288 on 592 blocks), one atomic per
// column per block took longer than reading the rows.
template <bool BF16, int MAXC, bool PREFETCH, bool REG>
__global__ void __launch_bounds__(ROW_THREADS)
calib_ln_absmax_kernel(const char* __restrict__ x, int64_t rows, int K, int64_t ld_bytes,
                       const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                       int rows_atomic, float* __restrict__ out) {
  extern __shared__ float colmax[];
  __shared__ float red[2 * (ROW_WARPS + 1)];
  const int nchunks = K / 8;
  float cm[REG ? MAXC * 8 : 1];
  if (REG) {
#pragma unroll
    for (int i = 0; i < MAXC * 8; ++i) cm[i] = 0.0f;
  } else if (!rows_atomic) {
    for (int j = threadIdx.x; j < K; j += ROW_THREADS) colmax[j] = 0.0f;
  }
  RowChunks<BF16, MAXC> rc;
  if ((int64_t)blockIdx.x < rows) rc.load(x + (int64_t)blockIdx.x * ld_bytes, nchunks);
  for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
    const int64_t rn = r + gridDim.x;
    RowChunks<BF16, MAXC> nxt;
    if (PREFETCH && rn < rows) nxt.load(x + rn * ld_bytes, nchunks);
    float mu, rstd;
    row_stats(rc, nchunks, K, eps, red, mu, rstd);
#pragma unroll
    for (int i = 0; i < MAXC; ++i) {
      const int c = threadIdx.x + i * ROW_THREADS;
      if (c < nchunks) {
        float f[8], y[8];
        rc.get(i, f);
        ln_chunk(f, mu, rstd, gamma, beta, c, y);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          if (REG) cm[i * 8 + e] = fmaxf(cm[i * 8 + e], fabsf(y[e]));
          else if (rows_atomic) atomic_max_nonneg(out + c * 8 + e, fabsf(y[e]));
          else colmax[c * 8 + e] = fmaxf(colmax[c * 8 + e], fabsf(y[e]));
        }
      }
    }
    if (PREFETCH) rc = nxt;
    else if (rn < rows) rc.load(x + rn * ld_bytes, nchunks);
  }
  if (REG) {
    if ((int64_t)blockIdx.x < rows) {
#pragma unroll
      for (int i = 0; i < MAXC; ++i) {
        const int c = threadIdx.x + i * ROW_THREADS;
        if (c < nchunks)
#pragma unroll
          for (int e = 0; e < 8; ++e) atomic_max_nonneg(out + c * 8 + e, cm[i * 8 + e]);
      }
    }
  } else if (!rows_atomic) {
    const uint32_t C = cluster_nctarank();
    if (C == 1) {
      __syncthreads();
      for (int j = threadIdx.x; j < K; j += ROW_THREADS) atomic_max_nonneg(out + j, colmax[j]);
    } else {
      cluster_sync();  // every block's maxima are complete (every block of the cluster gets here)
      const uint32_t q = cluster_ctarank();
      const int share = (K + (int)C - 1) / (int)C;
      const int j1 = min(K, (int)(q + 1) * share);
      for (int j = (int)q * share + threadIdx.x; j < j1; j += ROW_THREADS) {
        float m = colmax[j];
        for (uint32_t p = 0; p < C; ++p)
          if (p != q) m = fmaxf(m, ld_dsmem_f32(&colmax[j], p));
        atomic_max_nonneg(out + j, m);
      }
      cluster_sync();  // no block leaves while a peer still reads its shared memory
    }
  }
}

// Rows of up to 8192 elements: one group of T threads per row (see sq_rowln.cuh), the
// running column max of the thread's own chunks in registers across all rows the group
// visits, one atomicMax per column per group at the end.
// SMEM (T = 256, one row per block; rows of 12288 or 14336 over few tokens): the running
// maxima live in shared memory instead (48 or 56 KB), which leaves the registers for the
// prefetched next row at two blocks per SM; launched in clusters, the blocks of a cluster
// combine their maxima through distributed shared memory, and each column takes one atomicMax
// per cluster (one per block per column took longer than reading the rows).
constexpr int CALIB_CLUSTER = 8;

template <bool BF16, int T, int NCH, bool SMEM = false>
__global__ void __launch_bounds__(256)
calib_ln_group_kernel(const char* __restrict__ x, int64_t rows, int K, int64_t ld_bytes,
                      const float* __restrict__ gamma, const float* __restrict__ beta, float eps,
                      float* __restrict__ out) {
  static_assert(!SMEM || T == 256, "one row per block with the maxima in shared memory");
  constexpr int G = 256 / T;
  __shared__ float red[G][16];
  extern __shared__ float colsm[];  // SMEM: [K]
  const int gid = threadIdx.x / T, t = threadIdx.x % T;
  const int nchunks = K / 8;
  float cm[SMEM ? 1 : NCH * 8];
  if constexpr (SMEM) {
    for (int j = threadIdx.x; j < K; j += 256) colsm[j] = 0.0f;
  } else {
#pragma unroll
    for (int i = 0; i < NCH * 8; ++i) cm[i] = 0.0f;
  }
  RowRaw<BF16, NCH> raw;
  const int64_t rstep = (int64_t)gridDim.x * G;
  const int64_t r0 = (int64_t)blockIdx.x * G + gid;
  if (r0 < rows) raw.template load<T>(x + r0 * ld_bytes, nchunks, t);
  for (int64_t r = r0; r < rows; r += rstep) {
    float v[NCH * 8];
    raw.to_float(v);
    if (r + rstep < rows) raw.template load<T>(x + (r + rstep) * ld_bytes, nchunks, t);
    float mu, rstd;
    group_row_stats<T, NCH>(v, nchunks, K, eps, red[gid], t, gid, mu, rstd);
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = t + T * i;
      if (c < nchunks) {
        float y[8];
        ln_chunk(v + i * 8, mu, rstd, gamma, beta, c, y);
        if constexpr (SMEM) {
          float4* d = reinterpret_cast<float4*>(colsm + c * 8);  // this thread's own columns
          float4 a = d[0], b = d[1];
          a.x = fmaxf(a.x, fabsf(y[0])); a.y = fmaxf(a.y, fabsf(y[1]));
          a.z = fmaxf(a.z, fabsf(y[2])); a.w = fmaxf(a.w, fabsf(y[3]));
          b.x = fmaxf(b.x, fabsf(y[4])); b.y = fmaxf(b.y, fabsf(y[5]));
          b.z = fmaxf(b.z, fabsf(y[6])); b.w = fmaxf(b.w, fabsf(y[7]));
          d[0] = a;
          d[1] = b;
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) cm[i * 8 + e] = fmaxf(cm[i * 8 + e], fabsf(y[e]));
        }
      }
    }
  }
  if constexpr (SMEM) {
    const uint32_t C = cluster_nctarank();
    if (C == 1) {
      __syncthreads();
      if (r0 < rows)
        for (int j = threadIdx.x; j < K; j += 256) atomic_max_nonneg(out + j, colsm[j]);
    } else {
      // clusters of CALIB_CLUSTER blocks; K % (4 * CALIB_CLUSTER) == 0 on this route
      cluster_sync();  // every block's maxima are complete (every block of the cluster gets here)
      const uint32_t q = cluster_ctarank();
      const int share = K / CALIB_CLUSTER;
      for (int j = (int)q * share + 4 * threadIdx.x; j < (int)(q + 1) * share; j += 4 * 256) {
        float4 v[CALIB_CLUSTER];  // every CTA's four maxima, all loads in flight at once
#pragma unroll
        for (int p = 0; p < CALIB_CLUSTER; ++p) v[p] = ld_dsmem_f32x4(&colsm[j], (uint32_t)p);
        float4 m = v[0];
#pragma unroll
        for (int p = 1; p < CALIB_CLUSTER; ++p) {
          m.x = fmaxf(m.x, v[p].x); m.y = fmaxf(m.y, v[p].y);
          m.z = fmaxf(m.z, v[p].z); m.w = fmaxf(m.w, v[p].w);
        }
        atomic_max_nonneg(out + j, m.x);
        atomic_max_nonneg(out + j + 1, m.y);
        atomic_max_nonneg(out + j + 2, m.z);
        atomic_max_nonneg(out + j + 3, m.w);
      }
      cluster_sync();  // no block leaves while a peer still reads its shared memory
    }
  } else if (r0 < rows) {
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const int c = t + T * i;
      if (c < nchunks)
#pragma unroll
        for (int e = 0; e < 8; ++e) atomic_max_nonneg(out + c * 8 + e, cm[i * 8 + e]);
    }
  }
}

}  // namespace sqk

// ---------------------------------------------------------------------------- launchers
namespace sqh {

cudaError_t launch_absmax(const void* x, bool bf16, int64_t rows, int64_t cols, int64_t ld, int axis,
                          int accumulate, float* out, cudaStream_t st) {
  const int elt = bf16 ? 2 : 4;
  const int64_t nvec = cols * elt / 16;
  const int64_t ld_bytes = ld * elt;
  if (axis == 0) {
    if (!accumulate) {
      cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)cols, st);
      if (e != cudaSuccess) return e;
    }
    const int64_t gx = (nvec + sqk::COL_VX - 1) / sqk::COL_VX;
    const int64_t want = (int64_t)num_sms() * 8;  // 8 blocks of 256 threads per SM
    int64_t gy = std::max<int64_t>(1, want / gx);
    gy = std::min<int64_t>(gy, (rows + sqk::COL_RY - 1) / sqk::COL_RY);
    gy = std::min<int64_t>(gy, 65535);
    dim3 grid((unsigned)gx, (unsigned)gy), block(sqk::COL_VX, sqk::COL_RY);
    if (bf16)
      sqk::absmax_cols_kernel<true><<<grid, block, 0, st>>>((const char*)x, rows, nvec, ld_bytes, out);
    else
      sqk::absmax_cols_kernel<false><<<grid, block, 0, st>>>((const char*)x, rows, nvec, ld_bytes, out);
  } else if (nvec <= 32 * 16) {  // rows up to 8 KB: a warp per row
    const unsigned grid = (unsigned)((rows + 7) / 8);
#define SQ_RW(V)                                                                                                   \
  if (nvec <= 32 * V) {                                                                                            \
    if (bf16)                                                                                                      \
      sqk::absmax_rows_warp_kernel<true, V><<<grid, 256, 0, st>>>((const char*)x, rows, nvec, ld_bytes, accumulate, out); \
    else                                                                                                           \
      sqk::absmax_rows_warp_kernel<false, V><<<grid, 256, 0, st>>>((const char*)x, rows, nvec, ld_bytes, accumulate, out); \
    return cudaGetLastError();                                                                                     \
  }
    SQ_RW(2) SQ_RW(4) SQ_RW(8) SQ_RW(16)
#undef SQ_RW
  } else {
    if (bf16)
      sqk::absmax_rows_kernel<true><<<(unsigned)rows, 256, 0, st>>>((const char*)x, rows, nvec, ld_bytes, accumulate, out);
    else
      sqk::absmax_rows_kernel<false><<<(unsigned)rows, 256, 0, st>>>((const char*)x, rows, nvec, ld_bytes, accumulate, out);
  }
  return cudaGetLastError();
}

template <bool BF16, int MAXC>
static cudaError_t launch_calib_ln_t(const void* x, int64_t rows, int K, int64_t ld_bytes, const float* gamma,
                                     const float* beta, float eps, float* out, cudaStream_t st) {
  constexpr bool REG = MAXC <= 4;
  const size_t smem_cols = sizeof(float) * (size_t)K;
  const bool rows_atomic = !REG && smem_cols > 160 * 1024;
  const size_t smem = (REG || rows_atomic) ? 0 : smem_cols;
  auto kern = sqk::calib_ln_absmax_kernel<BF16, MAXC, BF16 && MAXC <= 4, REG>;
  {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  int per_sm = 1;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, sqk::ROW_THREADS, smem);
  if (e != cudaSuccess) return e;
  int64_t grid = std::min<int64_t>(rows, (int64_t)num_sms() * std::max(per_sm, 1));
  constexpr int CL = 8;  // blocks per cluster when the maxima are in shared memory
  if (REG || rows_atomic || grid < CL) {
    kern<<<(unsigned)grid, sqk::ROW_THREADS, smem, st>>>((const char*)x, rows, K, ld_bytes, gamma, beta, eps,
                                                         rows_atomic ? 1 : 0, out);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(sqk::ROW_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)(grid / CL * CL));
  int clusters = 0;
  e = max_active_clusters(reinterpret_cast<const void*>(kern), &cfg, &clusters);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3((unsigned)(CL * std::max<int64_t>(1, std::min<int64_t>(grid / CL, clusters))));
  return cudaLaunchKernelEx(&cfg, kern, (const char*)x, rows, K, ld_bytes, gamma, beta, eps, 0, out);
}

int pick_row_threads(int64_t K, int max_nch, int* nch);
bool rowpair_supported(int64_t K, bool bf16, bool calib, int64_t rows);
cudaError_t launch_rowpair_calib(const void* x, int64_t rows, int64_t K, int64_t ldx, const float* gamma,
                                 const float* beta, float eps, float* out, cudaStream_t st);
bool rowpipe_shape(int64_t K, bool bf16, int max_nch, int* T, int* nch);
cudaError_t launch_rowpipe_calib(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ldx, const float* gamma,
                                 const float* beta, float eps, float* out, int T, int nch, cudaStream_t st);

template <bool BF16, int T, int NCH>
static cudaError_t launch_calib_group_t(const void* x, int64_t rows, int K, int64_t ld_bytes, const float* gamma,
                                        const float* beta, float eps, float* out, cudaStream_t st) {
  auto kern = sqk::calib_ln_group_kernel<BF16, T, NCH>;
  int per_sm = 1;
  cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, 0);
  if (e != cudaSuccess) return e;
  constexpr int G = 256 / T;
  const int64_t blocks = (rows + G - 1) / G;
  const int64_t grid = std::min<int64_t>(blocks, (int64_t)num_sms() * std::max(per_sm, 1));
  kern<<<(unsigned)grid, 256, 0, st>>>((const char*)x, rows, K, ld_bytes, gamma, beta, eps, out);
  return cudaGetLastError();
}

// LayerNorm calibration of bf16 rows of 12288 or 14336 (6 or 7 chunks per thread) over few
// tokens: one row per block, maxima in shared memory, clusters of 8 blocks.
template <int NCH>
static cudaError_t launch_calib_smem_t(const void* x, int64_t rows, int K, int64_t ld_bytes, const float* gamma,
                                       const float* beta, float eps, float* out, cudaStream_t st) {
  auto kern = sqk::calib_ln_group_kernel<true, 256, NCH, true>;
  const size_t smem = sizeof(float) * (size_t)K;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int per_sm = 1;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, 256, smem);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(rows, (int64_t)num_sms() * std::max(per_sm, 1));
  constexpr int CL = sqk::CALIB_CLUSTER;
  if (grid < CL) {
    kern<<<(unsigned)grid, 256, smem, st>>>((const char*)x, rows, K, ld_bytes, gamma, beta, eps, out);
    return cudaGetLastError();
  }
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)(grid / CL * CL));
  int clusters = 0;
  e = max_active_clusters(reinterpret_cast<const void*>(kern), &cfg, &clusters);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3((unsigned)(CL * std::max<int64_t>(1, std::min<int64_t>(grid / CL, clusters))));
  return cudaLaunchKernelEx(&cfg, kern, (const char*)x, rows, K, ld_bytes, gamma, beta, eps, out);
}

template <bool BF16, int T>
static cudaError_t launch_calib_group_nch(int nch, const void* x, int64_t rows, int K, int64_t ld_bytes,
                                          const float* gamma, const float* beta, float eps, float* out,
                                          cudaStream_t st) {
  if (nch <= 1) return launch_calib_group_t<BF16, T, 1>(x, rows, K, ld_bytes, gamma, beta, eps, out, st);
  if (nch <= 2) return launch_calib_group_t<BF16, T, 2>(x, rows, K, ld_bytes, gamma, beta, eps, out, st);
  return launch_calib_group_t<BF16, T, 4>(x, rows, K, ld_bytes, gamma, beta, eps, out, st);
}

cudaError_t launch_calib_ln_absmax(const void* x, bool bf16, int64_t rows, int64_t K, int64_t ld,
                                   const float* gamma, const float* beta, float eps, int accumulate,
                                   float* out, cudaStream_t st) {
  if (!accumulate) {
    cudaError_t e = cudaMemsetAsync(out, 0, sizeof(float) * (size_t)K, st);
    if (e != cudaSuccess) return e;
  }
  const int64_t ldb = ld * (bf16 ? 2 : 4);
  if (rowpair_supported(K, bf16, true, rows))  // chunk-pair rows of the model widths
    return launch_rowpair_calib(x, rows, K, ld, gamma, beta, eps, out, st);
  if (bf16 && (K == 12288 || K == 14336)) {  // rows of the large model widths
    if (K == 12288) return launch_calib_smem_t<6>(x, rows, (int)K, ldb, gamma, beta, eps, out, st);
    return launch_calib_smem_t<7>(x, rows, (int)K, ldb, gamma, beta, eps, out, st);
  }
  int pT = 0, pn = 0;
  if (rowpipe_shape(K, bf16, 4, &pT, &pn))
    return launch_rowpipe_calib(x, bf16, rows, K, ld, gamma, beta, eps, out, pT, pn, st);
  int gnch = 0;
  const int T = pick_row_threads(K, 4, &gnch);
  if (T) {
    const int k = (int)K;
#define SQ_T(TT)                                                                                       \
  if (T == TT)                                                                                         \
    return bf16 ? launch_calib_group_nch<true, TT>(gnch, x, rows, k, ldb, gamma, beta, eps, out, st)   \
                : launch_calib_group_nch<false, TT>(gnch, x, rows, k, ldb, gamma, beta, eps, out, st);
    SQ_T(32) SQ_T(64) SQ_T(128) SQ_T(256)
#undef SQ_T
  }
  const int need = (int)((K / 8 + sqk::ROW_THREADS - 1) / sqk::ROW_THREADS);
  const int k = (int)K;
#define SQ_LN_CASE(C)                                                                                   \
  if (need <= C)                                                                                        \
    return bf16 ? launch_calib_ln_t<true, C>(x, rows, k, ldb, gamma, beta, eps, out, st)                \
                : launch_calib_ln_t<false, (C > 16 ? 16 : C)>(x, rows, k, ldb, gamma, beta, eps, out, st);
  SQ_LN_CASE(1) SQ_LN_CASE(2) SQ_LN_CASE(4) SQ_LN_CASE(8) SQ_LN_CASE(16) SQ_LN_CASE(24) SQ_LN_CASE(32)
#undef SQ_LN_CASE
  return cudaErrorInvalidValue;
}

}  // namespace sqh

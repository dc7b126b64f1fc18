// sq_gemm.cu -- INT8 x INT8 -> int32 GEMM with the SmoothQuant dequant epilogue on the
// 5th-generation (tcgen05) tensor cores of sm_100a, and its FP8 (E4M3 x E4M3 -> fp32)
// variant on the same pipeline (tcgen05.mma kind::f8f6f4).
//
//   acc[m, n] = sum_j xq[m, j] * wq[n, j]            exact int32 (FP8: fp32 accumulation)
//   y[m, n]   = bf16_rne(((float)acc * sx[m]) * sw[n])
//
// "4.2 W8A8 量化与 SmoothQuant" (intro, sec. 6): W8A8 lets the whole GEMM run on the INT8
// tensor cores and the runtime kernel is a plain INT8 GEMM; "量化：只压权重，与训练后量化
// （PTQ）", SmoothQuant section: per-token activation scales and per-output-channel weight
// scales are constant along the summed index, so they are applied after the GEMM.
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0      one lane issues TMA loads (128-byte swizzle, no multicast) of a 128-row
//               A tile and a BN-row B tile, 128 bytes of K each, into a STAGES-deep
//               shared-memory ring guarded by full/empty mbarriers;
//   warp 1      allocates TMEM; one lane issues tcgen05.mma.cta_group::1.kind::i8
//               (M = 128, N = BN, K = 32 per instruction) into one of two TMEM
//               accumulators, and tcgen05.commit frees ring slots / signals the epilogue;
//   warps 2-5   epilogue: tcgen05.ld of the int32 accumulator (warp w reads TMEM lanes
//               32*(w%4) .. +31), scale, convert, store; the second accumulator lets the
//               next tile's MMAs run meanwhile.
// Operands are K-major: A = xq [M, K], B = wq [N, K].  For decode-sized M (<= 128) the
// roles swap (A = wq, B = xq) so the weights fill the 128-row MMA dimension and the
// tokens the N dimension.  When the weight tiles do not fill the SMs evenly, the work is
// split stream-K style: the tiles' K blocks are laid end to end and every CTA takes an equal
// run of them, so a tile may be shared by a few CTAs; each adds its int32 partial tile into the
// tile's sum in the workspace, and a reduction kernel launched behind the GEMM (already
// resident, waiting on the GEMM grid) applies the epilogue to the shared tiles and puts their
// sums back to zero.  For M > 128 with fewer tiles than SMs, K is split and the same kind of
// second kernel sums the partials.
// Every mbarrier wait is bounded: on expiry the kernel records a code in a device error
// word and leaves.
#include <cuda.h>

#include <algorithm>
#include <cstddef>

#include "sq_ptx.cuh"

namespace sqk {

__device__ DeviceDiag g_diag = {0u, 0u, WAIT_NS};

constexpr int BM = 128;          // MMA M: rows of the A operand per tile
constexpr int BK = 128;          // K bytes per ring stage (one 128-byte swizzle row)
constexpr int UMMA_K = 32;       // K per tcgen05.mma kind::i8
constexpr int GEMM_THREADS = 192;

struct GemmParams {
  int tiles_a, tiles_b;      // tiles along A rows (BM) and B rows (BN)
  int num_kb;                // ceil(K / BK)
  int kb_per_split, splits;
  int num_units;             // tiles_a * tiles_b * splits
  int group_a;               // raster (b_major = 0): this many A tiles share a sweep over B tiles
  int group_b;               // raster (b_major = 1): this many B tiles share a sweep over A tiles
  int b_major;
  int keep;                  // CTA pairs: 1 = A tiles, 2 = B tiles loaded with an L2 evict-last hint, 0 = none
  int M, N;                  // output is y[M, N]
  const float* sx;
  const float* sw;
  void* y;
  int64_t ldy;
  int ydt;                   // SQ_BF16, SQ_F32 or SQ_I32
  int vec_store;             // y and every output row start on a 16-byte boundary
  int32_t* ws;               // [splits][M][N] int32 partials when splits > 1; with hy, the tail tiles' partials
  // split tail (CTA pairs): the first hy_dp tiles (whole waves) go whole; each of the hy_tail
  // remaining tiles is cut into hy_splits runs of hy_kbps K blocks, one unit each, whose
  // partial tiles go to ws as [hy_splits][hy_tail][256 rows][BN] int32 (FP8: fp32 bits)
  int hy, hy_dp, hy_tail, hy_splits, hy_kbps;
  // stream-K (swap layout only): the first sk_dp_tiles tiles go whole to the CTAs in full waves
  // (tile u to CTA u mod G); of the rest, CTA c of G = sk_ctas takes iterations
  // [c I / G, (c+1) I / G) of their I = (tiles_a - sk_dp_tiles) * num_kb (tile, K block)
  // iterations laid end to end
  int sk;
  int sk_ctas;
  int sk_dp_tiles;
  int64_t sk_iters;
  int32_t* partials;         // INT8: [tiles_a][BN][BM] int32 tile sums, zero at rest; FP8: [2 * sk_ctas][BN][BM]
                             // partial tiles, two slots per CTA (both column-major)
  float* rowmax;             // NULL, or [M]: running max over n of |y[m, n]| as stored (zeroed before the launch)
};

// TMA load whose completion is signalled on the mbarrier of the pair's leader CTA
// (`bar` is a shared::cluster address, e.g. from mapa).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

// The same with an L2 cache-policy hint (createpolicy): the operand that every wave reads
// again is kept in L2 ahead of the one that streams through.
__device__ __forceinline__ void tma_load_2d_pair_keep(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                                      uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
      : "memory");
}

// shared::cluster address of the same shared variable in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_shared(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

// Arrives on the same mbarrier in both CTAs of the pair when this thread's MMAs complete.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile(
      "{\n\t.reg .b16 m;\n\tmov.b16 m, 3;\n\t"
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], m;\n\t}" ::"r"(bar)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, both K-major, int8 -> int32 (F8: E4M3 -> fp32); CG = 2
// spans the CTA pair (M = 256, each CTA supplies 128 rows of A and half of B from the same
// smem offsets).
template <int CG, bool F8>
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                      uint32_t accumulate) {
  if (F8 && CG == 1)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else if (F8)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else if (CG == 1)
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
  else
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with 128-byte
// swizzle: rows of 128 bytes, 8-row swizzle atoms 1024 bytes apart (stride byte
// offset), leading byte offset unused for swizzled K-major layouts, descriptor version 1
// (sm_100), layout code 2 = 128-byte swizzle.  The tile base is 1024-byte aligned; the
// k-th 32-byte step inside a row advances the start address by 32 bytes.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;
  d |= (uint64_t)(1024 >> 4) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor of tcgen05.mma kind::i8: D = s32 (bits 4-5 = 2), A and B
// signed 8-bit (bits 7-9, 10-12 = 1), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n) {
  return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// Instruction descriptor of tcgen05.mma kind::f8f6f4 with E4M3 operands: D = f32 (bits 4-5
// = 1), A and B format E4M3 (code 0), both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t idesc_e4m3(int m, int n) {
  return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// 32 lanes x NCOL consecutive 32-bit TMEM columns -> NCOL registers per thread.
template <int NCOL>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, uint32_t* r);

template <>
__device__ __forceinline__ void tmem_ld<16>(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

template <>
__device__ __forceinline__ void tmem_ld<32>(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// The accumulator as binary32: an int32 rounded to nearest, or (F8) the fp32 bits as they are.
template <bool F8>
__device__ __forceinline__ float acc_value(uint32_t r) {
  return F8 ? __uint_as_float(r) : __int2float_rn((int32_t)r);
}

// Output value of one accumulator: ((float)acc * sx) * sw, each product rounded.
template <bool F8>
__device__ __forceinline__ float dequant(uint32_t acc, float sxm, float swn) {
  return __fmul_rn(__fmul_rn(acc_value<F8>(acc), sxm), swn);
}

// Stores one output and returns its magnitude as stored (the bf16 value for bf16 output; 0 for
// raw int32 output, which has no row max).
template <bool F8>
__device__ __forceinline__ float store_out(const GemmParams& p, int64_t m, int64_t n, uint32_t acc, float sxm,
                                           float swn) {
  const int64_t off = m * p.ldy + n;
  if (p.ydt == SQ_BF16) {
    const __nv_bfloat16 h = __float2bfloat16_rn(dequant<F8>(acc, sxm, swn));
    reinterpret_cast<__nv_bfloat16*>(p.y)[off] = h;
    return fabsf(__bfloat162float(h));
  }
  if (p.ydt == SQ_F32) {
    const float v = dequant<F8>(acc, sxm, swn);
    reinterpret_cast<float*>(p.y)[off] = v;
    return fabsf(v);
  }
  reinterpret_cast<int32_t*>(p.y)[off] = (int32_t)acc;
  return 0.0f;
}

// Max over the 32 lanes of a warp (every lane gets it).
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Unit u -> (A tile, B tile, K split).  Splits of one tile are adjacent so they run
// concurrently.  Tiles are rastered so that one operand stays resident in L2 while the
// other streams through once: a group of group_a A tiles sweeps over all B tiles (A tile
// index fastest), or, with b_major, a group of group_b B tiles sweeps over all A tiles.
__device__ __forceinline__ void tile_coords(const GemmParams& p, int tile, int& ta, int& tb) {
  if (!p.b_major) {
    const int group_size = p.group_a * p.tiles_b;
    const int group = tile / group_size;
    const int first_a = group * p.group_a;
    const int ga = min(p.tiles_a - first_a, p.group_a);
    const int in_group = tile % group_size;
    ta = first_a + in_group % ga;
    tb = in_group / ga;
  } else {
    const int group_size = p.group_b * p.tiles_a;
    const int group = tile / group_size;
    const int first_b = group * p.group_b;
    const int gb = min(p.tiles_b - first_b, p.group_b);
    const int in_group = tile % group_size;
    tb = first_b + in_group % gb;
    ta = in_group / gb;
  }
}

__device__ __forceinline__ void decode_unit(const GemmParams& p, int u, int& ta, int& tb, int& split) {
  split = u % p.splits;
  tile_coords(p, u / p.splits, ta, tb);
}

// The sequence of pieces (tile, K-block range) one CTA works on.  Data-parallel: units
// unit0, unit0 + step, ... (decode_unit).  Stream-K: the CTA's iteration range, cut at tile
// boundaries (the first and last piece may be partial tiles).
struct Work {
  int64_t it, end;  // stream-K cursor
  int u, step;      // data-parallel cursor
  int tail;         // split tail: index of the current piece's tile among the tail tiles, or -1
};

__device__ __forceinline__ Work work_begin(const GemmParams& p, int unit0, int unit_step) {
  Work w;
  w.u = unit0;
  w.step = unit_step;
  w.tail = -1;
  w.it = (int64_t)unit0 * p.sk_iters / p.sk_ctas;
  w.end = (int64_t)(unit0 + 1) * p.sk_iters / p.sk_ctas;
  return w;
}

__device__ __forceinline__ bool next_piece(const GemmParams& p, Work& w, int& ta, int& tb, int& kb0, int& kb1,
                                           int& split) {
  if (p.sk) {
    tb = 0;
    split = 0;
    if (w.u < p.sk_dp_tiles) {  // whole tiles of the full waves
      ta = w.u;
      kb0 = 0;
      kb1 = p.num_kb;
      w.u += w.step;
      return true;
    }
    if (w.it >= w.end) return false;
    const int t_rel = (int)(w.it / p.num_kb);
    ta = p.sk_dp_tiles + t_rel;
    kb0 = (int)(w.it - (int64_t)t_rel * p.num_kb);
    kb1 = (int)min((int64_t)p.num_kb, (int64_t)kb0 + (w.end - w.it));
    w.it += kb1 - kb0;
    return true;
  }
  if (w.u >= p.num_units) return false;
  if (p.hy) {
    const int u = w.u;
    w.u += w.step;
    if (u < p.hy_dp) {  // a whole tile of the full waves
      tile_coords(p, u, ta, tb);
      split = 0;
      kb0 = 0;
      kb1 = p.num_kb;
      w.tail = -1;
      return true;
    }
    const int v = u - p.hy_dp;
    w.tail = v / p.hy_splits;
    split = v % p.hy_splits;
    tile_coords(p, p.hy_dp + w.tail, ta, tb);
    kb0 = split * p.hy_kbps;
    kb1 = min(p.num_kb, kb0 + p.hy_kbps);
    return true;
  }
  decode_unit(p, w.u, ta, tb, split);
  kb0 = split * p.kb_per_split;
  kb1 = min(p.num_kb, kb0 + p.kb_per_split);
  w.u += w.step;
  return true;
}

// Stream-K bookkeeping over the split tiles (t_rel = tile - sk_dp_tiles): the CTA whose
// iteration range holds split iteration i, and the workspace slot of CTA c's piece of split
// tile t_rel (slot 2c: the piece in the tile where c's range starts; 2c + 1: where it ends --
// the only two pieces of a CTA that can be partial).
__device__ __forceinline__ int sk_owner(const GemmParams& p, int64_t i) {
  return (int)(((i + 1) * p.sk_ctas + p.sk_iters - 1) / p.sk_iters - 1);
}
__device__ __forceinline__ int sk_slot(const GemmParams& p, int c, int t_rel) {
  const int64_t first = (int64_t)c * p.sk_iters / p.sk_ctas;
  return 2 * c + ((int)(first / p.num_kb) == t_rel ? 0 : 1);
}

// Shared-memory layout of one CTA: BN_CTA rows of B per stage (BN / CG), BN accumulator
// columns per TMEM buffer.
template <int BN, int STAGES, int CG>
struct GemmSmem {
  static constexpr int BN_CTA = BN / CG;
  static constexpr int A_BYTES = BM * BK;
  static constexpr int B_BYTES = BN_CTA * BK;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int BAR_OFFSET = STAGES * STAGE_BYTES;
  static constexpr int NUM_BARS = 2 * STAGES + 4;
  static constexpr int TOTAL = 1024 /* alignment slack */ + BAR_OFFSET + NUM_BARS * 8 + 16;
  static constexpr int TMEM_COLS = (2 * BN < 32) ? 32 : 2 * BN;  // power of two for BN in {16..256}
};

// CG = 1: one CTA per output tile of 128 x BN.  CG = 2: a cluster of two CTAs per tile of
// 256 x BN; CTA r loads rows [128 r, 128 r + 128) of the A tile and [BN/2 r, BN/2 (r+1)) of
// the B tile, signalling the leader's (rank 0) full barrier; the leader issues the pair MMAs
// and its commits arrive on the barriers of both CTAs; each CTA's epilogue drains its own
// TMEM (its 128 rows x BN columns) and arrives on the leader's accumulator-empty barrier.
template <int BN, int STAGES, bool SWAP, int CG, bool F8>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
w8a8_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                 const GemmParams p) {
  using L = GemmSmem<BN, STAGES, CG>;
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "kind::i8 with M = 128 needs N % 16 == 0, 16..256");
  static_assert(CG == 1 || (!SWAP && BN % 32 == 0), "the pair path runs the non-swapped layout, N % 32 == 0");
  constexpr int MMA_M = BM * CG;
  constexpr uint32_t IDESC = F8 ? idesc_e4m3(MMA_M, BN) : idesc_i8(MMA_M, BN);
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t sbase = smem_u32(smem);
  const uint32_t bar0 = sbase + L::BAR_OFFSET;
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
  auto tfull_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + a); };
  auto tempty_bar = [&](int a) { return bar0 + 8u * (2 * STAGES + 2 + a); };
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(smem + L::BAR_OFFSET + L::NUM_BARS * 8);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;
  const bool leader = rank == 0;
  const int unit0 = blockIdx.x / CG, unit_step = gridDim.x / CG;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull_bar(a), 1);
      mbar_init(tempty_bar(a), 4 * CG);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_a)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&map_b)) : "memory");
  }
  if (warp == 1) {
    if (CG == 1) {
      asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                   "r"((uint32_t)L::TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    } else {
      asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_holder)),
                   "r"((uint32_t)L::TMEM_COLS)
                   : "memory");
      asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
  }
  tc_fence_before();
  if (CG == 2) cluster_sync();  // the peer's loads signal the leader's barriers: init first
  else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_holder);
  const unsigned long long limit = g_diag.wait_limit_ns;
  // Launched as a programmatic dependent of the previous kernel on the stream: the set-up above
  // overlaps its tail.  In the swap layout the weights are the streamed operand; an epilogue
  // warp (idle until the first accumulator) asks L2 for this CTA's first weight tiles before
  // waiting.  A prefetch only fills L2, the point of coherence, so it is safe even if the
  // previous kernel writes those weights: every read of the operands, scales and workspace
  // comes after the wait.
  if (SWAP && warp == 2 && lane == 0) {
    Work w = work_begin(p, unit0, unit_step);
    int ta, tb, kb0, kb1, split, n = 0;
    while (n < STAGES && next_piece(p, w, ta, tb, kb0, kb1, split))
      for (int kb = kb0; kb < kb1 && n < STAGES; ++kb, ++n) tma_prefetch_l2(&map_a, kb * BK, ta * BM);
  }
  asm volatile("griddepcontrol.wait;" ::: "memory");

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (each CTA)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      uint32_t issued = 0;  // bit s: stage s has been loaded; its last load used parity bit s of `par`
      uint32_t par = 0;
      uint64_t keep_policy = 0;
      if (CG == 2 && p.keep) asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(keep_policy));
      Work w = work_begin(p, unit0, unit_step);
      int ta, tb, kb0, kb1, split;
      while (ok && next_piece(p, w, ta, tb, kb0, kb1, split)) {
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, limit)) {
            atomicOr(&g_diag.error, ERR_GEMM_PRODUCER_WAIT);
            ok = false;
            break;
          }
          issued |= 1u << stage;
          par = (par & ~(1u << stage)) | (phase << stage);
          const uint32_t sa = sbase + stage * L::STAGE_BYTES;
          if (CG == 1) {
            mbar_arrive_expect_tx(full_bar(stage), (uint32_t)L::STAGE_BYTES);
            tma_load_2d(sa, &map_a, full_bar(stage), kb * BK, ta * BM);
            tma_load_2d(sa + L::A_BYTES, &map_b, full_bar(stage), kb * BK, tb * BN);
          } else {
            if (leader) mbar_arrive_expect_tx(full_bar(stage), (uint32_t)(CG * L::STAGE_BYTES));
            const uint32_t fb = map_shared(full_bar(stage), 0);
            const int ya = ta * MMA_M + (int)rank * BM, yb = tb * BN + (int)rank * L::BN_CTA;
            if (p.keep == 1) tma_load_2d_pair_keep(sa, &map_a, fb, kb * BK, ya, keep_policy);
            else tma_load_2d_pair(sa, &map_a, fb, kb * BK, ya);
            if (p.keep == 2) tma_load_2d_pair_keep(sa + L::A_BYTES, &map_b, fb, kb * BK, yb, keep_policy);
            else tma_load_2d_pair(sa + L::A_BYTES, &map_b, fb, kb * BK, yb);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // every load of this CTA is issued: the kernel launched behind this grid (the split
      // reduction, or the next GEMM) may be scheduled now; it waits for this grid's completion
      // before it reads anything
      asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
      if (!ok && leader) {
        // let the loads issued for this barrier land before the block exits (bounded, 100 ms)
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) (void)mbar_wait(full_bar(s), (par >> s) & 1u, DRAIN_NS);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      Work w = work_begin(p, unit0, unit_step);
      int ta, tb, kb0, kb1, split;
      for (; ok && next_piece(p, w, ta, tb, kb0, kb1, split); ++it) {
        const int acc = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(tempty_bar(acc), aph ^ 1u, limit)) {
          atomicOr(&g_diag.error, ERR_GEMM_MMA_WAIT);
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(full_bar(stage), phase, limit)) {
            atomicOr(&g_diag.error, ERR_GEMM_MMA_WAIT);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + stage * L::STAGE_BYTES;
          const uint32_t sb = sa + L::A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            tc_mma<CG, F8>(d_tmem, sw128_desc(sa + k * UMMA_K), sw128_desc(sb + k * UMMA_K), IDESC,
                          (kb > kb0 || k > 0) ? 1u : 0u);
          }
          if (CG == 1) tc_commit(empty_bar(stage));
          else tc_commit_pair(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (CG == 1) tc_commit(tfull_bar(acc));
        else tc_commit_pair(tfull_bar(acc));
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                 // TMEM lane quarter this warp may access
    const int row = q * 32 + lane;          // row of this CTA's A tile = TMEM lane
    int it = 0;
    Work w = work_begin(p, unit0, unit_step);
    int ta, tb, kb0, kb1, split;
    for (; next_piece(p, w, ta, tb, kb0, kb1, split); ++it) {
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      if (!mbar_wait(tfull_bar(acc), aph, limit)) {
        atomicOr(&g_diag.error, ERR_GEMM_EPILOGUE_WAIT);
        break;
      }
      __syncwarp();  // tcgen05.ld below is .sync.aligned: reconverge after the wait loop
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int64_t arow = (int64_t)ta * MMA_M + (int64_t)rank * BM + row;
      constexpr int CH = BN >= 32 ? 32 : 16;
      float rmax = 0.0f;  // this thread's output row: max |y| over the tile's columns (rowmax mode)
      if (SWAP && p.sk && !(kb0 == 0 && kb1 == p.num_kb)) {
        // ---- a partial tile (stream-K): INT8 adds it into the tile's int32 sum (exact in any
        // order), FP8 writes it to this CTA's slot; the reduction kernel that follows this grid
        // finishes the tile
        const int t_rel = ta - p.sk_dp_tiles;
        int32_t* dst = p.partials + (int64_t)(F8 ? sk_slot(p, (int)blockIdx.x, t_rel) : t_rel) * (BM * BN) + row;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += CH) {
          uint32_t r[CH];
          tmem_ld<CH>(taddr + (uint32_t)c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            if (F8) __stcg(dst + (c0 + i) * BM, (int)r[i]);
            else atomicAdd(dst + (c0 + i) * BM, (int)r[i]);  // return value unused: a reduction
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(tempty_bar(acc));
        continue;
      }
      if (!SWAP && p.hy && w.tail >= 0) {
        // ---- a piece of a split tail tile: the raw partial (int32, or fp32 bits) into its slot;
        // the reduction kernel that follows this grid sums the pieces in split order
        int32_t* dst = p.ws + (((int64_t)split * p.hy_tail + w.tail) * MMA_M + (int64_t)rank * BM + row) * BN;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += CH) {
          uint32_t r[CH];
          tmem_ld<CH>(taddr + (uint32_t)c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < CH; i += 4)
            *reinterpret_cast<uint4*>(dst + c0 + i) = make_uint4(r[i], r[i + 1], r[i + 2], r[i + 3]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 1) mbar_arrive(tempty_bar(acc));
          else mbar_arrive_cluster(map_shared(tempty_bar(acc), 0));
        }
        continue;
      }
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += CH) {
        uint32_t r[CH];
        tmem_ld<CH>(taddr + (uint32_t)c0, r);
        tmem_wait_ld();
        if (!SWAP) {
          // A row = output row m; TMEM columns = output columns n
          const int64_t m = arow;
          const int64_t n0 = (int64_t)tb * BN + c0;
          if (m < p.M && n0 < p.N) {
            if (p.splits > 1) {
              int32_t* dst = p.ws + ((int64_t)split * p.M + m) * p.N + n0;
              for (int i = 0; i < CH; ++i)
                if (n0 + i < p.N) dst[i] = (int32_t)r[i];
            } else {
              const float sxm = p.ydt == SQ_I32 ? 0.0f : __ldg(p.sx + m);
              const bool full = n0 + CH <= p.N && p.vec_store;
              if (full && p.ydt == SQ_BF16) {
                uint32_t packed[CH / 2];
#pragma unroll
                for (int i = 0; i < CH; i += 2) {
                  const float v0 = dequant<F8>(r[i], sxm, __ldg(p.sw + n0 + i));
                  const float v1 = dequant<F8>(r[i + 1], sxm, __ldg(p.sw + n0 + i + 1));
                  __nv_bfloat162 h = __halves2bfloat162(__float2bfloat16_rn(v0), __float2bfloat16_rn(v1));
                  packed[i / 2] = *reinterpret_cast<uint32_t*>(&h);
                  rmax = fmax3(rmax, fabsf(__low2float(h)), fabsf(__high2float(h)));
                }
                uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.y) + m * p.ldy + n0);
#pragma unroll
                for (int v = 0; v < CH / 8; ++v)
                  dst[v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
              } else if (full && p.ydt == SQ_F32) {
                float4* dst = reinterpret_cast<float4*>(reinterpret_cast<float*>(p.y) + m * p.ldy + n0);
#pragma unroll
                for (int v = 0; v < CH / 4; ++v) {  // (sw is only 4-byte aligned: scalar loads)
                  const float* w = p.sw + n0 + 4 * v;
                  const float4 o = make_float4(dequant<F8>(r[4 * v], sxm, __ldg(w)), dequant<F8>(r[4 * v + 1], sxm, __ldg(w + 1)),
                                               dequant<F8>(r[4 * v + 2], sxm, __ldg(w + 2)),
                                               dequant<F8>(r[4 * v + 3], sxm, __ldg(w + 3)));
                  dst[v] = o;
                  rmax = fmax3(rmax, fmax3(fabsf(o.x), fabsf(o.y), fabsf(o.z)), fabsf(o.w));
                }
              } else {
                for (int i = 0; i < CH; ++i) {
                  const int64_t n = n0 + i;
                  if (n < p.N) rmax = fmaxf(rmax, store_out<F8>(p, m, n, r[i], sxm, p.ydt == SQ_I32 ? 0.0f : __ldg(p.sw + n)));
                }
              }
            }
          }
        } else {
          // A row = output column n; TMEM columns = output rows m
          const int64_t n = arow;
          const int64_t m0 = (int64_t)tb * BN + c0;
          // (swap-layout tiles are whole here: partial ones took the stream-K branch)
          const float swn = (p.ydt == SQ_I32 || n >= p.N) ? 0.0f : __ldg(p.sw + n);
          for (int i = 0; i < CH; ++i) {
            const int64_t m = m0 + i;
            float a = 0.0f;
            if (m < p.M && n < p.N) a = store_out<F8>(p, m, n, r[i], p.ydt == SQ_I32 ? 0.0f : __ldg(p.sx + m), swn);
            if (p.rowmax) {  // output row m spans the lanes (one output column n per lane)
              a = warp_max(a);
              if (lane == 0 && m < p.M) atomic_max_nonneg(p.rowmax + m, a);
            }
          }
        }
      }
      if (!SWAP && p.rowmax && p.splits == 1 && arow < p.M) atomic_max_nonneg(p.rowmax + arow, rmax);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (CG == 1) mbar_arrive(tempty_bar(acc));
        else mbar_arrive_cluster(map_shared(tempty_bar(acc), 0));
      }
    }
  }

  tc_fence_before();
  if (CG == 2) cluster_sync();  // no CTA of the pair leaves while its peer may still use it
  else __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    if (CG == 1)
      asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"((uint32_t)L::TMEM_COLS)
                   : "memory");
    else
      asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base),
                   "r"((uint32_t)L::TMEM_COLS)
                   : "memory");
  }
}


// Sums the split-K partials in split order (int32: exact; F8: fp32 in that fixed order),
// applies the epilogue and zeroes the partials (the workspace is zero at rest).
template <bool F8>
__global__ void __launch_bounds__(256)
splitk_reduce_kernel(int32_t* __restrict__ ws, int splits, int64_t M, int64_t N, const float* __restrict__ sx,
                     const float* __restrict__ sw, void* __restrict__ y, int64_t ldy, int ydt, float* rowmax) {
  // launched as a programmatic dependent of the GEMM: its blocks may be resident before the
  // GEMM ends, and wait here until the GEMM grid has completed and its partials are visible
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int64_t total = M * N;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
    uint32_t acc;
    if (F8) {
      float a = 0.0f;
      for (int s = 0; s < splits; ++s) a = __fadd_rn(a, __int_as_float(ws[(int64_t)s * total + i]));
      acc = __float_as_uint(a);
    } else {
      int32_t a = 0;
      for (int s = 0; s < splits; ++s) a += ws[(int64_t)s * total + i];
      acc = (uint32_t)a;
    }
    for (int s = 0; s < splits; ++s) ws[(int64_t)s * total + i] = 0;
    const int64_t m = i / N, n = i % N;
    const int64_t off = m * ldy + n;
    if (ydt == SQ_BF16) {
      const __nv_bfloat16 h = __float2bfloat16_rn(dequant<F8>(acc, __ldg(sx + m), __ldg(sw + n)));
      reinterpret_cast<__nv_bfloat16*>(y)[off] = h;
      if (rowmax) atomic_max_nonneg(rowmax + m, fabsf(__bfloat162float(h)));
    } else if (ydt == SQ_F32) {
      const float v = dequant<F8>(acc, __ldg(sx + m), __ldg(sw + n));
      reinterpret_cast<float*>(y)[off] = v;
      if (rowmax) atomic_max_nonneg(rowmax + m, fabsf(v));
    } else {
      reinterpret_cast<int32_t*>(y)[off] = (int32_t)acc;
    }
  }
}

// Finishes the split tail tiles of a CTA-pair GEMM: y = epilogue(sum of the pieces in split
// order: int32 exact, FP8 fp32 in that fixed order), the row maxima for rowmax, and the pieces
// back to zero.  Thread: four consecutive columns of one row of one tail tile.
template <bool F8>
__global__ void __launch_bounds__(256)
hy_reduce_kernel(const GemmParams p, int bn) {
  allow_dependent_launch();
  asm volatile("griddepcontrol.wait;" ::: "memory");  // the GEMM grid has completed
  const int per_tile = 256 * bn / 4;                  // 4-column groups of one tail tile
  const int64_t total = (int64_t)p.hy_tail * per_tile;
  const int64_t slab = (int64_t)p.hy_tail * 256 * bn;  // one split's pieces
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    const int t = (int)(g / per_tile), e = (int)(g % per_tile);
    const int r = e / (bn / 4), c = (e % (bn / 4)) * 4;
    int ta, tb;
    tile_coords(p, p.hy_dp + t, ta, tb);
    const int64_t m = (int64_t)ta * 256 + r, n0 = (int64_t)tb * bn + c;
    int32_t* src = p.ws + ((int64_t)t * 256 + r) * bn + c;
    uint32_t acc[4];
    if (F8) {
      float a[4] = {0.f, 0.f, 0.f, 0.f};
      for (int s = 0; s < p.hy_splits; ++s) {
        const uint4 v = *reinterpret_cast<const uint4*>(src + s * slab);
        a[0] = __fadd_rn(a[0], __uint_as_float(v.x)); a[1] = __fadd_rn(a[1], __uint_as_float(v.y));
        a[2] = __fadd_rn(a[2], __uint_as_float(v.z)); a[3] = __fadd_rn(a[3], __uint_as_float(v.w));
        *reinterpret_cast<uint4*>(src + s * slab) = make_uint4(0u, 0u, 0u, 0u);
      }
      for (int i = 0; i < 4; ++i) acc[i] = __float_as_uint(a[i]);
    } else {
      int32_t a[4] = {0, 0, 0, 0};
      for (int s = 0; s < p.hy_splits; ++s) {
        const int4 v = *reinterpret_cast<const int4*>(src + s * slab);
        a[0] += v.x; a[1] += v.y; a[2] += v.z; a[3] += v.w;
        *reinterpret_cast<int4*>(src + s * slab) = make_int4(0, 0, 0, 0);
      }
      for (int i = 0; i < 4; ++i) acc[i] = (uint32_t)a[i];
    }
    if (m >= p.M) continue;
    const float sxm = p.ydt == SQ_I32 ? 0.0f : __ldg(p.sx + m);
    float rmax = 0.0f;
    for (int i = 0; i < 4; ++i) {
      const int64_t n = n0 + i;
      if (n < p.N) rmax = fmaxf(rmax, store_out<F8>(p, m, n, acc[i], sxm, p.ydt == SQ_I32 ? 0.0f : __ldg(p.sw + n)));
    }
    if (p.rowmax) atomic_max_nonneg(p.rowmax + m, rmax);
  }
}

// Finishes the tiles of a stream-K GEMM that several CTAs shared: y = epilogue(sum of the
// partial tiles), and the workspace back to zero.  INT8: the int32 tile sum; FP8: the
// contributors' slots added in K order.  Block b covers 1024 elements of split tile b / (BN / 8)
// (column-major inside the tile): each thread four consecutive rows n of one column m.
template <bool F8>
__global__ void __launch_bounds__(256)
sk_reduce_kernel(const GemmParams p, int bn) {
  // the next kernel on the stream may start its set-up now; this grid's work waits for the GEMM
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int chunks = bn / 8;  // BM * bn / 1024
  const int t_rel = (int)(blockIdx.x / chunks);
  const int c_first = sk_owner(p, (int64_t)t_rel * p.num_kb);
  const int c_last = sk_owner(p, (int64_t)(t_rel + 1) * p.num_kb - 1);
  if (c_first == c_last) return;  // a whole tile: the GEMM stored it
  const int per_tile = BM * bn;
  const int e = (int)(blockIdx.x % chunks) * 1024 + threadIdx.x * 4;  // element of the tile
  const int col = e / BM, row = e % BM;
  uint32_t acc[4];
  if (!F8) {
    int4* a = reinterpret_cast<int4*>(p.partials + (int64_t)t_rel * per_tile + e);
    const int4 v = __ldcg(a);
    __stcg(a, make_int4(0, 0, 0, 0));
    acc[0] = (uint32_t)v.x; acc[1] = (uint32_t)v.y; acc[2] = (uint32_t)v.z; acc[3] = (uint32_t)v.w;
  } else {
    float sum[4] = {0.0f, 0.0f, 0.0f, 0.0f};
    for (int c = c_first; c <= c_last; ++c) {
      int4* a = reinterpret_cast<int4*>(p.partials + (int64_t)sk_slot(p, c, t_rel) * per_tile + e);
      const int4 v = __ldcg(a);
      __stcg(a, make_int4(0, 0, 0, 0));
      sum[0] = __fadd_rn(sum[0], __int_as_float(v.x));
      sum[1] = __fadd_rn(sum[1], __int_as_float(v.y));
      sum[2] = __fadd_rn(sum[2], __int_as_float(v.z));
      sum[3] = __fadd_rn(sum[3], __int_as_float(v.w));
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[i] = __float_as_uint(sum[i]);
  }
  const int64_t m = col;  // the same for the 32 lanes of a warp (32 x 4 rows = one column of the tile)
  if (m >= p.M) return;
  const float sxm = p.ydt == SQ_I32 ? 0.0f : __ldg(p.sx + m);
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t n = (int64_t)(p.sk_dp_tiles + t_rel) * BM + row + i;
    if (n < p.N) a = fmaxf(a, store_out<F8>(p, m, n, acc[i], sxm, p.ydt == SQ_I32 ? 0.0f : __ldg(p.sw + n)));
  }
  if (p.rowmax) {
    a = warp_max(a);
    if ((threadIdx.x & 31) == 0) atomic_max_nonneg(p.rowmax + m, a);
  }
}

}  // namespace sqk

// ============================================================================= host side
namespace sqh {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool make_tmap_2d(CUtensorMap* map, bool two_byte, const void* base, int64_t inner, int64_t outer,
                  int64_t row_bytes, int box_inner, int box_outer, bool swizzle128) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, two_byte ? CU_TENSOR_MAP_DATA_TYPE_UINT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
            const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D int8 tensor [rows, K] (K contiguous) tiled as box_rows x 128 bytes, 128-byte swizzle,
// zero fill outside the tensor.
static bool make_map(CUtensorMap* map, const void* base, int64_t rows, int64_t K, int box_rows) {
  return make_tmap_2d(map, false, base, K, rows, K, sqk::BK, box_rows, true);
}

// Launch plan for one GEMM shape on the current device.
struct GemmPlan {
  bool swap;
  int cg;  // CTAs per MMA tile (2: a CTA pair computes 256-row tiles)
  int bn;
  int tiles_a, tiles_b, num_kb, kb_per_split, splits;
  bool sk;          // stream-K split of the swap layout
  int sk_ctas, sk_dp_tiles;
  int64_t sk_iters;
  bool hy;          // split tail of the CTA-pair layout
  int hy_dp, hy_tail, hy_splits, hy_kbps;
  size_t ws_bytes;  // 0, or the split-K partials / stream-K tile sums / split-tail pieces (zero at rest)
};

// split_tail = false: the plan without the split tail (which is the only part of a CTA-pair
// plan with many tiles that needs a workspace).
static GemmPlan plan_gemm(int64_t M, int64_t N, int64_t K, bool split_tail = true) {
  GemmPlan pl{};
  const int sms = num_sms();
  pl.swap = M <= 128;
  pl.cg = 1;
  pl.num_kb = (int)((K + sqk::BK - 1) / sqk::BK);
  if (pl.swap) {
    pl.bn = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
    pl.tiles_a = (int)((N + sqk::BM - 1) / sqk::BM);
    pl.tiles_b = 1;
    pl.splits = 1;
    pl.kb_per_split = pl.num_kb;
    // Weight streaming: every SM should stream the same number of bytes.  Whole tiles per CTA
    // when they fill the SMs within 10%; otherwise stream-K, at least 4 K blocks (64 KB of
    // weights) per CTA.
    const int64_t tiles = pl.tiles_a;
    const int64_t waves = (tiles + sms - 1) / sms;
    if (tiles * 10 < waves * sms * 9) {
      // whole tiles in the full waves, stream-K over the remaining tiles
      pl.sk = true;
      pl.sk_dp_tiles = (int)(tiles / sms * sms);
      const int64_t split_tiles = tiles - pl.sk_dp_tiles;
      pl.sk_iters = split_tiles * pl.num_kb;
      pl.sk_ctas = pl.sk_dp_tiles ? sms : (int)std::min<int64_t>(sms, std::max<int64_t>(1, pl.sk_iters / 4));
      // int32 tile sums (INT8) or two partial slots per CTA (FP8), whichever is larger
      const int64_t tiles_or_slots = std::max<int64_t>(split_tiles, 2 * (int64_t)pl.sk_ctas);
      pl.ws_bytes = (size_t)tiles_or_slots * sqk::BM * pl.bn * sizeof(int32_t);
    }
    return pl;
  }
  // CTA-pair tiles of 256 x 256 (192-column tiles, which fill the waves better on some shapes,
  // measured slower: 221 against 199 us at 2048 x 12288 x 12288, 161 against 134 at 8192 x 6144 x 4096)
  pl.bn = 256;
  pl.cg = 2;
  const int64_t tile_m = (int64_t)sqk::BM * pl.cg;
  pl.tiles_a = (int)((M + tile_m - 1) / tile_m);
  pl.tiles_b = (int)((N + pl.bn - 1) / pl.bn);
  const int64_t tiles = (int64_t)pl.tiles_a * pl.tiles_b;
  const int slots = sms / pl.cg;  // tiles that run at once
  int splits = 1;
  if (tiles < slots) {
    splits = (int)std::max<int64_t>(1, slots / tiles);
    splits = std::min(splits, std::max(1, pl.num_kb / 4));
  }
  pl.kb_per_split = (pl.num_kb + splits - 1) / splits;
  pl.splits = (pl.num_kb + pl.kb_per_split - 1) / pl.kb_per_split;
  pl.ws_bytes = pl.splits > 1 ? (size_t)pl.splits * (size_t)M * (size_t)N * sizeof(int32_t) : 0;
  // Split tail: when the last wave holds at most half as many tiles as there are CTA pairs,
  // its tiles are cut along K so that all pairs share it; the full waves keep whole tiles.
  // Only for long K (pieces of at least 64 K blocks): 2048 x 12288 x 49152 (5 waves of 74
  // tiles and 14) measured 734 against 780 us, while pieces of 16-20 K blocks cost more than
  // the short wave they save (2048 x 12288 x 12288: 202 against 200 us; 8192 x 6144 x 4096:
  // 160-179 against 138-142 us): a piece writes a whole 256 x 256 partial tile.
  if (split_tail && tiles >= slots) {
    const int64_t tail = tiles % slots;
    const int64_t hs = tail ? std::min<int64_t>(slots / tail, pl.num_kb / 64) : 0;
    if (hs >= 2) {
      pl.hy = true;
      pl.hy_dp = (int)(tiles - tail);
      pl.hy_tail = (int)tail;
      pl.hy_kbps = (int)((pl.num_kb + hs - 1) / hs);
      pl.hy_splits = (pl.num_kb + pl.hy_kbps - 1) / pl.hy_kbps;
      pl.ws_bytes = (size_t)pl.hy_splits * (size_t)tail * tile_m * (size_t)pl.bn * sizeof(int32_t);
    }
  }
  return pl;
}

size_t gemm_workspace_size(int64_t M, int64_t N, int64_t K) { return plan_gemm(M, N, K).ws_bytes; }
// The smallest workspace a launch of this shape can run with (no split tail).
size_t gemm_workspace_size_min(int64_t M, int64_t N, int64_t K) { return plan_gemm(M, N, K, false).ws_bytes; }

template <int BN, int STAGES, bool SWAP, int CG, bool F8>
static cudaError_t launch_cfg(const CUtensorMap& ma, const CUtensorMap& mb, const sqk::GemmParams& p,
                              cudaStream_t st) {
  using L = sqk::GemmSmem<BN, STAGES, CG>;
  auto kern = sqk::w8a8_gemm_kernel<BN, STAGES, SWAP, CG, F8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::TOTAL);
  if (e != cudaSuccess) return e;
  const int slots = num_sms() / CG;
  const int grid = p.sk ? p.sk_ctas : std::min(p.num_units, slots) * CG;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(sqk::GEMM_THREADS);
  cfg.dynamicSmemBytes = L::TOTAL;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  // programmatic dependent launch: the CTAs' set-up may overlap the previous kernel's tail
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = CG;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = CG == 1 ? 1 : 2;
  return cudaLaunchKernelEx(&cfg, kern, ma, mb, p);
}

template <bool F8>
static cudaError_t launch_gemm_any(const void* xq, const float* sx, const void* wq, const float* sw, int64_t M,
                                   int64_t N, int64_t K, void* y, int ydt, int64_t ldy, void* ws, size_t ws_bytes,
                                   float* rowmax, cudaStream_t st, bool* ws_too_small) {
  GemmPlan pl = plan_gemm(M, N, K);
  // a workspace too small for the split tail: the plan without it (which needs none)
  if (pl.hy && (ws == nullptr || ws_bytes < pl.ws_bytes)) pl = plan_gemm(M, N, K, false);
  *ws_too_small = pl.ws_bytes > 0 && (ws == nullptr || ws_bytes < pl.ws_bytes);
  if (*ws_too_small) return cudaSuccess;
  if (rowmax) {  // the epilogue takes a running max into it
    const cudaError_t ez = cudaMemsetAsync(rowmax, 0, sizeof(float) * (size_t)M, st);
    if (ez != cudaSuccess) return ez;
  }
  CUtensorMap ma, mb;
  const void* a_ptr = pl.swap ? (const void*)wq : (const void*)xq;
  const void* b_ptr = pl.swap ? (const void*)xq : (const void*)wq;
  const int64_t a_rows = pl.swap ? N : M;
  const int64_t b_rows = pl.swap ? M : N;
  if (!make_map(&ma, a_ptr, a_rows, K, sqk::BM) || !make_map(&mb, b_ptr, b_rows, K, pl.bn / pl.cg))
    return cudaErrorInvalidValue;
  sqk::GemmParams p{};
  p.tiles_a = pl.tiles_a;
  p.tiles_b = pl.tiles_b;
  p.num_kb = pl.num_kb;
  p.kb_per_split = pl.kb_per_split;
  p.splits = pl.splits;
  p.num_units = pl.hy ? pl.hy_dp + pl.hy_tail * pl.hy_splits : pl.tiles_a * pl.tiles_b * pl.splits;
  p.hy = pl.hy ? 1 : 0;
  p.hy_dp = pl.hy_dp;
  p.hy_tail = pl.hy_tail;
  p.hy_splits = pl.hy ? pl.hy_splits : 1;
  p.hy_kbps = pl.hy_kbps;
  // Tile order: the smaller operand's tiles are the fast index within a group, so the tiles
  // one wave runs at once (they step through K together) share each K-block of both operands
  // through L2.  A smaller operand of at most 64 MB forms one group and stays in L2 for the
  // whole sweep (its loads carry an evict-last hint on CTA pairs); the larger one streams
  // through once.  A larger smaller operand is taken about sqrt(CTA pairs) tiles at a time
  // (square waves read the fewest tiles per wave).  Measured DRAM reads at 2048 x 12288 x
  // 49152 with groups sized for 48 MB of L2: 2.74 GB for 0.70 GB of operands.
  {
    const int64_t a_bytes = (pl.swap ? N : M) * K, b_bytes = (pl.swap ? M : N) * K;
    const int64_t resident = 64ll << 20;
    const int64_t pairs = num_sms() / pl.cg;  // tiles that run at once
    int64_t side = 1;
    while (side * side < pairs) ++side;
    if (a_bytes <= b_bytes) {
      p.b_major = 0;
      p.group_a = (int)(a_bytes <= resident ? pl.tiles_a : std::min<int64_t>(pl.tiles_a, side));
      p.group_b = 1;
      p.keep = (pl.cg == 2 && a_bytes <= resident) ? 1 : 0;
    } else {
      p.b_major = 1;
      p.group_b = (int)(b_bytes <= resident ? pl.tiles_b : std::min<int64_t>(pl.tiles_b, side));
      p.group_a = 1;
      p.keep = (pl.cg == 2 && b_bytes <= resident) ? 2 : 0;
    }
  }
  p.M = (int)M;
  p.N = (int)N;
  p.sx = sx;
  p.sw = sw;
  p.y = y;
  p.ldy = ldy;
  p.ydt = ydt;
  const int64_t elt = ydt == SQ_BF16 ? 2 : 4;
  p.vec_store = (reinterpret_cast<uintptr_t>(y) % 16 == 0) && (ldy * elt) % 16 == 0;
  // workspace (zero at rest): split-K partials, or the stream-K tile sums / slots
  p.ws = pl.ws_bytes ? static_cast<int32_t*>(ws) : nullptr;
  p.partials = p.ws;
  p.sk = pl.sk ? 1 : 0;
  p.sk_ctas = pl.sk ? pl.sk_ctas : 1;
  p.sk_dp_tiles = pl.sk ? pl.sk_dp_tiles : 0;
  p.sk_iters = pl.sk ? pl.sk_iters : 1;
  p.rowmax = rowmax;
  cudaError_t e;
  if (!pl.swap) {
    e = launch_cfg<256, 6, false, 2, F8>(ma, mb, p, st);
  } else {
    switch (pl.bn) {
      case 16: e = launch_cfg<16, 10, true, 1, F8>(ma, mb, p, st); break;
      case 32: e = launch_cfg<32, 9, true, 1, F8>(ma, mb, p, st); break;
      case 64: e = launch_cfg<64, 8, true, 1, F8>(ma, mb, p, st); break;
      default: e = launch_cfg<128, 6, true, 1, F8>(ma, mb, p, st); break;
    }
  }
  if (e != cudaSuccess) return e;
  if (pl.sk) {
    // the shared tiles' reduction, a programmatic dependent of the GEMM (resident while it runs)
    const int64_t blocks = (int64_t)(pl.tiles_a - pl.sk_dp_tiles) * (pl.bn / 8);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)blocks);
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, sqk::sk_reduce_kernel<F8>, p, pl.bn);
  }
  if (pl.hy) {
    // the split tail's reduction, a programmatic dependent of the GEMM
    const int64_t groups = (int64_t)pl.hy_tail * 256 * pl.bn / 4;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)std::min<int64_t>((groups + 255) / 256, (int64_t)num_sms() * 8));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, sqk::hy_reduce_kernel<F8>, p, pl.bn);
  }
  if (pl.splits == 1) return e;
  const int64_t total = M * N;
  const int64_t grid = std::min<int64_t>((total + 255) / 256, (int64_t)num_sms() * 16);
  // programmatic dependent launch: the reduction's launch overlaps the GEMM's tail
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(256);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, sqk::splitk_reduce_kernel<F8>, p.ws, pl.splits, M, N, sx, sw, y, ldy, ydt, rowmax);
}

cudaError_t launch_gemm(const int8_t* xq, const float* sx, const int8_t* wq, const float* sw, int64_t M, int64_t N,
                        int64_t K, void* y, int ydt, int64_t ldy, void* ws, size_t ws_bytes, float* rowmax,
                        cudaStream_t st, bool* ws_too_small) {
  return launch_gemm_any<false>(xq, sx, wq, sw, M, N, K, y, ydt, ldy, ws, ws_bytes, rowmax, st, ws_too_small);
}

// FP8 variant: E4M3 codes, fp32 accumulation, the same epilogue (ydt BF16 or F32).
cudaError_t launch_gemm_fp8(const uint8_t* xq, const float* sx, const uint8_t* wq, const float* sw, int64_t M,
                            int64_t N, int64_t K, void* y, int ydt, int64_t ldy, void* ws, size_t ws_bytes,
                            cudaStream_t st, bool* ws_too_small) {
  return launch_gemm_any<true>(xq, sx, wq, sw, M, N, K, y, ydt, ldy, ws, ws_bytes, nullptr, st, ws_too_small);
}

// Device address of the error word on the current device (for kernels in other files).
unsigned int* error_word_ptr() {
  static unsigned int* ptrs[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, sqk::g_diag) == cudaSuccess) ptrs[dev] = static_cast<unsigned int*>(p);
  }
  return ptrs[dev];
}

cudaError_t read_device_error(unsigned int* code, int clear, cudaStream_t st) {
  cudaError_t e = cudaMemcpyFromSymbolAsync(code, sqk::g_diag, sizeof(unsigned int), 0, cudaMemcpyDeviceToHost, st);
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess || !clear) return e;
  const unsigned int zero = 0;
  e = cudaMemcpyToSymbolAsync(sqk::g_diag, &zero, sizeof(unsigned int), 0, cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

cudaError_t set_wait_limit(unsigned long long ns, cudaStream_t st) {
  cudaError_t e = cudaMemcpyToSymbolAsync(sqk::g_diag, &ns, sizeof(ns), offsetof(sqk::DeviceDiag, wait_limit_ns),
                                          cudaMemcpyHostToDevice, st);
  if (e != cudaSuccess) return e;
  return cudaStreamSynchronize(st);
}

}  // namespace sqh

// gemm.cuh -- steps 4, 5 and 6 for prefill shapes on the 5th-generation tensor cores.
//
//   acc[t,n]  = sum_k Xq[t,k] * CB[n,k]                     tcgen05.mma kind::i8 (int32, TMEM)
//   D[t,n]    = acc[t,n] * SCx[t]/127                       epilogue, written back to TMEM (fp32)
//   D[t,n]   += sum_j X_o[t,j] * CB_o[n,j]                  tcgen05.mma kind::f16 on top of D
//   C[t,n]    = fp16(D[t,n] * SCB[n]/127 + bias[n])         epilogue
//
// Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at
// scale" (Hugging Face blog), "内部的 MatMul": the int8 product of row-quantised hidden
// states and column-quantised weights, dequantised and added to the fp16 product of the
// outlier columns; "absmax 量化": dequantisation by the outer product of the absmax
// vectors; "用法": the fp16 weights of the outlier product are CB * SCB / 127.
//
// Design (sm_100a): persistent clusters of two CTAs on an SM pair, 256 x 256 output tiles,
// tcgen05.mma.cta_group::2 (M = 256: each CTA holds 128 rows of A and 128 rows of B in its
// own shared memory, and 128 rows x 256 columns of the accumulator in its own TMEM).
//   warps 0, 6  TMA producers (both CTAs; warp 0 loads A, warp 6 loads B): 128 B of K per
//               stage, 128-byte swizzle, no multicast; both CTAs' loads complete on the
//               leader CTA's barrier.  B_o comes from one of two tensor maps (the
//               workspace's CB_o slice, or an outlier cache's), chosen by a device word.
//   warp 1      TMEM allocation (both CTAs); the leader's lane 0 issues every MMA and
//               commits with multicast to both CTAs' barriers.
//   warps 2..5  epilogue (both CTAs): tcgen05.ld / tcgen05.st, per-column scales staged in
//               shared memory, fp16 stores.  Warp w reads TMEM lanes 32*(w%4)..+31.
// TMEM holds two 256-column accumulators, so the epilogue of one tile always overlaps the
// MMAs of the next.  With outlier columns, the int32 accumulator of tile i is converted in
// place to fp32 (times SCx/127) by the epilogue, and the fp16 outlier MMAs of tile i,
// issued after the first few K-blocks of tile i+1, accumulate on top of it.
// FP8 variant (kE4M3): e4m3 codes, tcgen05.mma kind::f8f6f4 with an fp32 accumulator that
// the epilogue reads as it is, and 448 in place of 127 in both scales.
#pragma once

#include "common.cuh"

namespace i8 {
namespace gemm {

constexpr int TM = 256;        // cluster tile rows (tokens)
constexpr int TN = 256;        // cluster tile columns (output features)
constexpr int HM = TM / 2;     // rows of A per CTA
constexpr int HN = TN / 2;     // rows of B per CTA
constexpr int BK = 128;        // bytes of K per stage
constexpr int STAGES = 6;
constexpr int A_BYTES = HM * BK;
constexpr int B_BYTES = HN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // per CTA
constexpr int THREADS = 224;     // warps 0,6 TMA (A, B); 1 MMA; 2..5 epilogue
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_I8 = idesc_s8_s32(TM, TN);
constexpr uint32_t IDESC_F16 = idesc_f16_f32(TM, TN);
constexpr uint32_t IDESC_E4M3 = idesc_e4m3_f32(TM, TN);
constexpr int INSERT_AT = 8;    // K-blocks of tile i+1 issued before the outlier MMAs of tile i
                                // (at least; a quarter of the K-blocks in longer K-loops, so
                                // that tile i's conversion has finished by then)
constexpr int GROUP_M = 16;     // m-tiles per raster group (L2 reuse of Xq)
constexpr int COL_BYTES = 2 * 2 * TN * 4;        // SCB/127 and bias as fp32, two buffers
// fp16 output staging for the TMA stores of C: per epilogue warp two 32 x 32 blocks
constexpr int CST_BYTES = 4 * 2 * 32 * 64;
constexpr int BAR_BYTES = 256;
constexpr size_t SMEM_BYTES =
    static_cast<size_t>(STAGES) * STAGE_BYTES + COL_BYTES + CST_BYTES + BAR_BYTES + 1024;
constexpr uint16_t PAIR_MASK = 0x3;

static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");
static_assert(THREADS == 224, "warp roles assume 7 warps");

struct Args {
  int T, N, K;
  int m_tiles, n_tiles, k_blocks;
  const int32_t* n_outliers;  // device scalar, NULL = no outlier phase
  const int32_t* cbo_sel;     // device scalar or NULL: nonzero = B_o comes from tmBc
  const float* SCx;
  const float* SCB;
  const __half* bias;  // nullable
  __half* C;
  int32_t* acc_out;  // raw-accumulator mode
  bool c_tma;        // C is written by TMA stores through tmC (N % 8 == 0), else by threads
  uint64_t wait_limit_ns;
};

struct SmemBars {
  uint64_t full[STAGES];     // leader: TMA bytes of both CTAs landed
  uint64_t empty[STAGES];    // both: MMAs reading the slot are done
  uint64_t int_full[2];      // both: int8 MMAs of the buffer's tile are done
  uint64_t tmem_full[2];     // both: the buffer's tile is final
  uint64_t converted[2];     // leader: both epilogues converted the buffer to fp32
  uint64_t tmem_empty[2];    // leader: both epilogues released the buffer
  uint64_t drain;            // leader: every issued MMA is done
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(SmemBars) <= BAR_BYTES, "barrier block");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}

// shared::cluster address of the same offset in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t map_to_rank(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}

__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* m,
                                                 uint32_t leader_bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(leader_bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* m,
                                                 uint32_t leader_bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(leader_bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void umma_i8_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_e4m3_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on the barrier at `bar` in both CTAs of the pair when every tcgen05 op
// issued so far by this thread is done.
__device__ __forceinline__ void umma_commit_pair(uint32_t bar) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(bar),
      "h"(PAIR_MASK)
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void epilogue_bar() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// An accumulator word as fp32: an int32 sum of int8 products, or already fp32 (e4m3).
template <bool kE4M3>
__device__ __forceinline__ float acc_value(uint32_t r) {
  return kE4M3 ? __uint_as_float(r) : static_cast<float>(static_cast<int32_t>(r));
}

// fp32 outputs of one 32-column chunk of a row from its accumulator words: with outlier
// MMAs the words already hold acc*SCx/127 + the outlier product (fp32); without, the raw
// accumulator (int32, or fp32 for e4m3) is scaled here.  Then * SCB/127 (/448) + bias.
template <bool kE4M3>
__device__ __forceinline__ void epilogue_values(const uint32_t (&r)[32], int OC, float sx,
                                                const float* wsc, const float* bsc,
                                                float (&v)[32]) {
  if (OC > 0) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = fmaf(__uint_as_float(r[j]), wsc[j], bsc[j]);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = fmaf(acc_value<kE4M3>(r[j]) * sx, wsc[j], bsc[j]);
  }
}

__device__ __forceinline__ void sts_v4(uint32_t addr, uint32_t x, uint32_t y, uint32_t z,
                                       uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(x), "r"(y), "r"(z),
               "r"(w)
               : "memory");
}

// TMA store of a shared-memory box to global memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, uint32_t src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(src), "r"(x), "r"(y)
               : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// wait until at most the most recent bulk group still reads its shared-memory source
__device__ __forceinline__ void bulk_wait_read_1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}

__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// this thread's generic-proxy shared-memory writes become visible to the async proxy
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Stores 32 consecutive fp16 outputs of one row (c0 = first column of the chunk).
__device__ __forceinline__ void store_row32_f16(__half* crow, int c0, int N, const float (&v)[32],
                                                bool vec_ok) {
  if (vec_ok && c0 + 32 <= N) {
    uint4* dst = reinterpret_cast<uint4*>(crow + c0);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      __half2 h0 = __floats2half2_rn(v[8 * q + 0], v[8 * q + 1]);
      __half2 h1 = __floats2half2_rn(v[8 * q + 2], v[8 * q + 3]);
      __half2 h2 = __floats2half2_rn(v[8 * q + 4], v[8 * q + 5]);
      __half2 h3 = __floats2half2_rn(v[8 * q + 6], v[8 * q + 7]);
      uint4 u;
      u.x = *reinterpret_cast<uint32_t*>(&h0);
      u.y = *reinterpret_cast<uint32_t*>(&h1);
      u.z = *reinterpret_cast<uint32_t*>(&h2);
      u.w = *reinterpret_cast<uint32_t*>(&h3);
      dst[q] = u;
    }
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (c0 + j < N) crow[c0 + j] = __float2half_rn(v[j]);
  }
}

// The order in which both the producer and the MMA issuer walk the shared-memory ring:
// for each local tile, its int8 K-blocks; the outlier chunks of the previous tile are
// slotted in after INSERT_AT K-blocks (or after the last one), and those of the final
// tile come last.  `visit(kind, tile_slot, idx)` is called per ring stage with kind 0 =
// int8 K-block idx of local tile tile_slot, kind 1 = outlier chunk idx of tile_slot, and
// kind 2 / 3 marking the start / end of a tile's int8 phase (no ring stage).
template <class F>
__device__ __forceinline__ bool walk_schedule(int L, int KB, int OC, F&& visit) {
  const int ins = KB < INSERT_AT ? KB : (KB / 4 > INSERT_AT ? KB / 4 : INSERT_AT);
  for (int it = 0; it < L; ++it) {
    if (!visit(2, it, 0)) return false;
    for (int kb = 0; kb < KB; ++kb) {
      if (OC > 0 && it > 0 && kb == ins)
        for (int c = 0; c < OC; ++c)
          if (!visit(1, it - 1, c)) return false;
      if (!visit(0, it, kb)) return false;
    }
    if (OC > 0 && it > 0 && ins >= KB)
      for (int c = 0; c < OC; ++c)
        if (!visit(1, it - 1, c)) return false;
    if (!visit(3, it, 0)) return false;
  }
  if (OC > 0 && L > 0)
    for (int c = 0; c < OC; ++c)
      if (!visit(1, L - 1, c)) return false;
  return true;
}

// kRaw: write the int32 accumulators (int8 codes only).  kE4M3: the codes are e4m3
// (kind::f8f6f4, fp32 accumulators, scales over 448) instead of int8 (kind::i8, int32
// accumulators, scales over 127).
template <bool kRaw, bool kE4M3 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    i8_gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmAo,
                           const __grid_constant__ CUtensorMap tmBo,
                           const __grid_constant__ CUtensorMap tmBc,
                           const __grid_constant__ CUtensorMap tmC, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t ring = raw_s + pad;  // 1024-aligned shared address of stage 0
  float* colbuf = reinterpret_cast<float*>(smem + static_cast<size_t>(STAGES) * STAGE_BYTES);
  const uint32_t cstage = ring + static_cast<uint32_t>(STAGES * STAGE_BYTES + COL_BYTES);
  SmemBars* bars = reinterpret_cast<SmemBars*>(smem + static_cast<size_t>(STAGES) * STAGE_BYTES +
                                               COL_BYTES + CST_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->int_full[b]), 1);
      mbar_init(smem_u32(&bars->tmem_full[b]), 1);
      mbar_init(smem_u32(&bars->converted[b]), 8);   // 4 epilogue warps x 2 CTAs
      mbar_init(smem_u32(&bars->tmem_empty[b]), 8);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmAo);
    tma_prefetch_desc(&tmBo);
    tma_prefetch_desc(&tmBc);
    if (a.c_tma) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&bars->tmem_base), TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;
  constexpr float kInvQ = kE4M3 ? 1.0f / 448.0f : 1.0f / 127.0f;
  // everything above overlaps the previous kernel; its outputs are read from here on
  grid_dep_wait();

  const int n_o = (a.n_outliers != nullptr) ? max(0, __ldg(a.n_outliers)) : 0;
  const int OC = (n_o + 63) >> 6;
  const int KB = a.k_blocks;
  const int num_tiles = a.m_tiles * a.n_tiles;
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;
  const int L = cluster_id < num_tiles ? (num_tiles - 1 - cluster_id) / num_clusters + 1 : 0;
  const uint64_t lim = a.wait_limit_ns;

  // Grouped raster: consecutive tiles walk GROUP_M m-tiles, then the next n-tile, so the
  // tiles in flight share a block of Xq rows and a few CB row blocks that fit in L2.
  const int G = a.m_tiles < GROUP_M ? a.m_tiles : GROUP_M;
  auto tile_mn = [&](int it, int& m0, int& n0) {
    const int t = cluster_id + it * num_clusters;
    const int group = t / (G * a.n_tiles);
    const int r = t - group * (G * a.n_tiles);
    const int mb = group * G;
    const int rows = (a.m_tiles - mb) < G ? (a.m_tiles - mb) : G;
    m0 = (mb + r % rows) * TM;
    n0 = (r / rows) * TN;
  };
  auto tile_m0 = [&](int it) {
    int m0, n0;
    tile_mn(it, m0, n0);
    return m0;
  };
  auto tile_n0 = [&](int it) {
    int m0, n0;
    tile_mn(it, m0, n0);
    return n0;
  };

  if (warp == 0 || warp == 6) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producers
      // Warp 0 loads the A (Xq / X_o) half of every stage and arms the leader's barrier
      // for both halves; warp 6 loads the B (CB / CB_o) half.  Splitting the issue over
      // two warps halves the per-stage latency chain of each issuing thread.
      const bool loads_a = (warp == 0);
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      int coord_it[2] = {-1, -1};
      int coord[2] = {0, 0};
      const uint32_t full_leader0 = map_to_rank(smem_u32(&bars->full[0]), 0);
      const CUtensorMap* map_i = loads_a ? &tmA : &tmB;
      // the prepare pass wrote the selector before this grid's dependency wait returned
      const bool b_cached = !loads_a && a.cbo_sel != nullptr && __ldcg(a.cbo_sel) != 0;
      const CUtensorMap* map_o = loads_a ? &tmAo : (b_cached ? &tmBc : &tmBo);
      const uint32_t half_off = loads_a ? 0u : static_cast<uint32_t>(A_BYTES);
      const bool ok = walk_schedule(L, KB, OC, [&](int kind, int it, int idx) -> bool {
        if (kind >= 2) return true;
        const int slot = it & 1;
        if (coord_it[slot] != it) {
          int m0, n0;
          tile_mn(it, m0, n0);
          coord[slot] = (loads_a ? m0 : n0) + static_cast<int>(rank) * (loads_a ? HM : HN);
          coord_it[slot] = it;
        }
        if (!mbar_wait(smem_u32(&bars->empty[s]), ph ^ 1u, abort_flag, lim)) return false;
        const uint32_t dst = ring + s * STAGE_BYTES + half_off;
        if (loads_a && rank == 0) mbar_arrive_expect_tx(smem_u32(&bars->full[s]), 2 * STAGE_BYTES);
        const uint32_t fb = full_leader0 + static_cast<uint32_t>(s) * 8u;
        if (kind == 0)
          tma_load_2d_pair(dst, map_i, fb, idx * BK, coord[slot]);
        else
          tma_load_3d_pair(dst, map_o, fb, 0, coord[slot], idx);
        ++issued;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
        return true;
      });
      if (!ok && loads_a && rank == 0) {
        // wind down: wait (bounded, ignoring the abort flag) for the copies in flight
        int no_abort = 0;
        const uint32_t inflight = issued < STAGES ? issued : STAGES;
        for (uint32_t i = 0; i < inflight; ++i) {
          const uint32_t u = issued - 1 - i;
          mbar_wait(smem_u32(&bars->full[u % STAGES]), (u / STAGES) & 1u, &no_abort, lim);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------------ MMA issuer (leader)
      int s = 0;
      uint32_t ph = 0;
      int conv_wait_done = -1;  // last tile whose conversion barrier was consumed
      walk_schedule(L, KB, OC, [&](int kind, int it, int idx) -> bool {
        const int b = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (kind == 2) {  // start of tile it's int8 phase: its buffer must be free
          if (!mbar_wait(smem_u32(&bars->tmem_empty[b]), (use & 1u) ^ 1u, abort_flag, lim))
            return false;
          tc_fence_after();
          return true;
        }
        if (kind == 3) {  // end of tile it's int8 phase
          umma_commit_pair(smem_u32(OC > 0 ? &bars->int_full[b] : &bars->tmem_full[b]));
          return true;
        }
        if (kind == 1 && conv_wait_done != it) {  // first outlier chunk of tile it
          if (!mbar_wait(smem_u32(&bars->converted[b]), use & 1u, abort_flag, lim)) return false;
          tc_fence_after();
          conv_wait_done = it;
        }
        if (!mbar_wait(smem_u32(&bars->full[s]), ph, abort_flag, lim)) return false;
        tc_fence_after();
        const uint32_t sa = ring + s * STAGE_BYTES;
        const uint32_t sb = sa + A_BYTES;
        const uint32_t d = tmem_base + static_cast<uint32_t>(b * TN);
        if (kind == 0 && kE4M3) {
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            umma_e4m3_pair(d, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32),
                           IDESC_E4M3, (idx | kk) != 0);
        } else if (kind == 0) {
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            umma_i8_pair(d, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32), IDESC_I8,
                         (idx | kk) != 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < BK / 32; ++kk)
            umma_f16_pair(d, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32), IDESC_F16,
                          1u);
        }
        umma_commit_pair(smem_u32(&bars->empty[s]));
        if (kind == 1 && idx == OC - 1) umma_commit_pair(smem_u32(&bars->tmem_full[b]));
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
        return true;
      });
      // every MMA issued by this thread completes before TMEM is released
      int no_abort = 0;
      umma_commit_pair(smem_u32(&bars->drain));
      mbar_wait(smem_u32(&bars->drain), 0u, &no_abort, lim);
    }
  } else if (warp >= 2 && warp <= 5) {
    // -------------------------------------------------------------- epilogue warps
    const int q = warp & 3;
    const int et = threadIdx.x - 64;  // 0..127 among the epilogue threads
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const bool vec_ok = (a.N % 8) == 0;
    // A warp that gives up on a wait keeps walking the tiles (it must still meet the
    // other epilogue warps at every named barrier) but touches TMEM no more.
    bool dead = false;
    int cbuf = 0;  // this warp's C staging buffer for the next TMA store
    for (int it = 0; it < L; ++it) {
      const int b = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      const int m0 = tile_m0(it);
      const int n0 = tile_n0(it);
      const int trow0 = m0 + static_cast<int>(rank) * HM + q * 32;  // the warp's first row
      const int t = trow0 + lane;
      const bool row_ok = t < a.T;
      float* ws = colbuf + b * (2 * TN);
      float* bs = ws + TN;
      if (!kRaw) {
        for (int j = et; j < TN; j += 128) {
          const int n = n0 + j;
          ws[j] = n < a.N ? __ldg(a.SCB + n) * kInvQ : 0.0f;
          bs[j] = (n < a.N && a.bias) ? __half2float(a.bias[n]) : 0.0f;
        }
      }
      epilogue_bar();
      if (dead) continue;
      const float sx = (!kRaw && row_ok) ? __ldg(a.SCx + t) * kInvQ : 0.0f;
      const uint32_t tb = lane_base + static_cast<uint32_t>(b * TN);

      if (!kRaw && OC > 0) {
        // accumulator (int32, or fp32 for e4m3) -> fp32 * SCx/127 (/448) in place; the
        // outlier MMAs then add on top
        bool got = mbar_wait(smem_u32(&bars->int_full[b]), use & 1u, abort_flag, lim);
        if (!__all_sync(0xffffffffu, got)) {
          dead = true;
          continue;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < TN / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tb + static_cast<uint32_t>(c * 32), r);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j)
            r[j] = __float_as_uint(acc_value<kE4M3>(r[j]) * sx);
          tmem_st_32x32b_x32(tb + static_cast<uint32_t>(c * 32), r);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_remote(map_to_rank(smem_u32(&bars->converted[b]), 0));
      }
      {
        bool got = mbar_wait(smem_u32(&bars->tmem_full[b]), use & 1u, abort_flag, lim);
        if (!__all_sync(0xffffffffu, got)) {
          dead = true;
          continue;
        }
      }
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < TN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tb + static_cast<uint32_t>(c * 32), r);
        tmem_ld_wait();
        const int c0 = n0 + c * 32;
        if (row_ok && c0 < a.N) {
          if (kRaw) {
            int32_t* arow = a.acc_out + static_cast<int64_t>(t) * a.N;
            if ((a.N % 4) == 0 && c0 + 32 <= a.N) {
              uint4* dst = reinterpret_cast<uint4*>(arow + c0);
#pragma unroll
              for (int j = 0; j < 8; ++j)
                dst[j] = make_uint4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (c0 + j < a.N) arow[c0 + j] = static_cast<int32_t>(r[j]);
            }
          } else if (!a.c_tma) {
            float v[32];
            epilogue_values<kE4M3>(r, OC, sx, ws + c * 32, ws + TN + c * 32, v);
            store_row32_f16(a.C + static_cast<int64_t>(t) * a.N, c0, a.N, v, vec_ok);
          }
        }
        if (!kRaw && a.c_tma && c0 < a.N && trow0 < a.T) {
          // the warp's 32 rows x 32 columns in fp16 through shared memory, one TMA store
          // (rows past T and columns past N are clipped by the tensor map)
          float v[32];
          epilogue_values<kE4M3>(r, OC, sx, ws + c * 32, ws + TN + c * 32, v);
          const uint32_t sb = cstage + static_cast<uint32_t>((q * 2 + cbuf) * 2048);
          if (lane == 0) bulk_wait_read_1();  // the store that last read this buffer is done
          __syncwarp();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            __half2 h0 = __floats2half2_rn(v[8 * q4 + 0], v[8 * q4 + 1]);
            __half2 h1 = __floats2half2_rn(v[8 * q4 + 2], v[8 * q4 + 3]);
            __half2 h2 = __floats2half2_rn(v[8 * q4 + 4], v[8 * q4 + 5]);
            __half2 h3 = __floats2half2_rn(v[8 * q4 + 6], v[8 * q4 + 7]);
            sts_v4(sb + static_cast<uint32_t>(lane * 64 + q4 * 16),
                   *reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                   *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_2d(&tmC, sb, c0, trow0);
            bulk_commit();
          }
          cbuf ^= 1;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_remote(map_to_rank(smem_u32(&bars->tmem_empty[b]), 0));
    }
    // the shared-memory reads and global writes of this warp's TMA stores are complete
    // before the CTA can exit
    if (lane == 0) bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  cluster_sync();
}

}  // namespace gemm
}  // namespace i8

// gemm_wide.cuh -- steps 4, 5 and 6 for prefill shapes with long K-loops: the products and
// epilogue of gemm.cuh on 256 x 512 output tiles per pair of CTAs.
//
//   acc[t,n]  = sum_k Xq[t,k] * CB[n,k]                     tcgen05.mma kind::i8 (int32, TMEM)
//   D[t,n]    = acc[t,n] * SCx[t]/127                       epilogue, written back to TMEM (fp32)
//   D[t,n]   += sum_j X_o[t,j] * CB_o[n,j]                  tcgen05.mma kind::f16 on top of D
//   C[t,n]    = fp16(D[t,n] * SCB[n]/127 + bias[n])         epilogue
//
// Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at
// scale" (Hugging Face blog), "内部的 MatMul", "absmax 量化" and "用法" (as gemm.cuh).
//
// Why a second tile shape: the 256 x 256 kernel is bound by each SM's operand feed (TMA
// issue and the SM's L2 port), not by the tensor pipe.  Here every K-step issues two
// M = 256, N = 256 pair MMAs that share the A tile: per CTA and stage 16 KB of A and 32 KB
// of B (two 128-row boxes) feed twice the work of the 32 KB stage of gemm.cuh, a quarter
// fewer operand bytes and TMA copies per multiply-add.  The price: the accumulator takes
// all 512 TMEM columns, so a tile's epilogue (and, with outlier columns, its conversion
// pass) no longer overlaps the next tile's MMAs; with long K-loops that is a few percent.
//
// Roles as in gemm.cuh: warp 0 loads A (and arms the leader's barrier), warp 6 loads B,
// warp 1 allocates TMEM and (leader lane 0) issues the MMAs, warps 2..5 run the epilogue.
// The outlier chunks of a tile follow its int8 K-blocks in the ring.  kE4M3: e4m3 codes
// (kind::f8f6f4, fp32 accumulator, scales over 448).
#pragma once

#include "common.cuh"
#include "gemm.cuh"

namespace i8 {
namespace gemmw {

using gemm::BK;
using gemm::HM;
using gemm::TM;
constexpr int TN = 512;                           // cluster tile columns
constexpr int HN = 128;                           // rows of one B box
constexpr int STAGES = 4;
constexpr int A_BYTES = HM * BK;                  // 16 KB
constexpr int B_BYTES = 2 * HN * BK;              // 32 KB: two boxes
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // 48 KB per CTA
constexpr int THREADS = 224;
constexpr uint32_t TMEM_COLS = 512;
constexpr int GROUP_M = 16;
constexpr int COL_BYTES = 2 * 2 * TN * 4;         // SCB/127 and bias, two buffers
constexpr int CST_BYTES = 4 * 2 * 32 * 64;        // fp16 C staging, two 32x32 blocks per warp
constexpr int BAR_BYTES = 256;
constexpr size_t SMEM_BYTES =
    static_cast<size_t>(STAGES) * STAGE_BYTES + COL_BYTES + CST_BYTES + BAR_BYTES + 1024;
constexpr uint32_t IDESC_I8 = idesc_s8_s32(TM, 256);
constexpr uint32_t IDESC_F16 = idesc_f16_f32(TM, 256);
constexpr uint32_t IDESC_E4M3 = idesc_e4m3_f32(TM, 256);

static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

struct SmemBars {
  uint64_t full[STAGES];     // leader: TMA bytes of both CTAs landed
  uint64_t empty[STAGES];    // both: MMAs reading the slot are done
  uint64_t int_full;         // both: int8 MMAs of the tile are done
  uint64_t tmem_full;        // both: the tile is final
  uint64_t converted;        // leader: both epilogues converted the tile to fp32
  uint64_t tmem_empty;       // leader: both epilogues released the accumulator
  uint64_t drain;            // leader: every issued MMA is done
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(SmemBars) <= BAR_BYTES, "barrier block");

template <bool kE4M3 = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    i8_gemm_wide_kernel(const __grid_constant__ CUtensorMap tmA,
                        const __grid_constant__ CUtensorMap tmB,
                        const __grid_constant__ CUtensorMap tmAo,
                        const __grid_constant__ CUtensorMap tmBo,
                        const __grid_constant__ CUtensorMap tmBc,
                        const __grid_constant__ CUtensorMap tmC, const gemm::Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t ring = raw_s + pad;
  float* colbuf = reinterpret_cast<float*>(smem + static_cast<size_t>(STAGES) * STAGE_BYTES);
  const uint32_t cstage = ring + static_cast<uint32_t>(STAGES * STAGE_BYTES + COL_BYTES);
  SmemBars* bars = reinterpret_cast<SmemBars*>(smem + static_cast<size_t>(STAGES) * STAGE_BYTES +
                                               COL_BYTES + CST_BYTES);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = gemm::cluster_rank();
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    mbar_init(smem_u32(&bars->int_full), 1);
    mbar_init(smem_u32(&bars->tmem_full), 1);
    mbar_init(smem_u32(&bars->converted), 8);   // 4 epilogue warps x 2 CTAs
    mbar_init(smem_u32(&bars->tmem_empty), 8);
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
    gemm::tmem_alloc_pair(smem_u32(&bars->tmem_base), TMEM_COLS);
    gemm::tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  gemm::cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;
  constexpr float kInvQ = kE4M3 ? 1.0f / 448.0f : 1.0f / 127.0f;
  grid_dep_wait();   // the prepare pass's outputs are read from here on

  const int n_o = (a.n_outliers != nullptr) ? max(0, __ldg(a.n_outliers)) : 0;
  const int OC = (n_o + 63) >> 6;
  const int KB = a.k_blocks;
  const int num_tiles = a.m_tiles * a.n_tiles;
  const int cluster_id = blockIdx.x >> 1;
  const int num_clusters = gridDim.x >> 1;
  const int L = cluster_id < num_tiles ? (num_tiles - 1 - cluster_id) / num_clusters + 1 : 0;
  const uint64_t lim = a.wait_limit_ns;
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

  if (warp == 0 || warp == 6) {
    if (lane == 0) {
      // ---------------------------------------------------------------- TMA producers
      // Per tile: KB int8 stages, then OC outlier stages.  Warp 0 loads A (Xq / X_o) and
      // arms the leader's barrier for both CTAs' bytes; warp 6 loads the two B boxes.
      const bool loads_a = (warp == 0);
      const bool b_cached = !loads_a && a.cbo_sel != nullptr && __ldcg(a.cbo_sel) != 0;
      const CUtensorMap* map_i = loads_a ? &tmA : &tmB;
      const CUtensorMap* map_o = loads_a ? &tmAo : (b_cached ? &tmBc : &tmBo);
      const uint32_t half_off = loads_a ? 0u : static_cast<uint32_t>(A_BYTES);
      const uint32_t full_leader0 = gemm::map_to_rank(smem_u32(&bars->full[0]), 0);
      int s = 0;
      uint32_t ph = 0, issued = 0;
      bool ok = true;
      for (int it = 0; it < L && ok; ++it) {
        int m0, n0;
        tile_mn(it, m0, n0);
        const int ca = m0 + static_cast<int>(rank) * HM;         // A rows of this CTA
        const int cb0 = n0 + static_cast<int>(rank) * HN;        // B rows of box 0
        const int cb1 = n0 + 256 + static_cast<int>(rank) * HN;  // B rows of box 1
        for (int st = 0; st < KB + OC && ok; ++st) {
          if (!mbar_wait(smem_u32(&bars->empty[s]), ph ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          const uint32_t dst = ring + s * STAGE_BYTES + half_off;
          if (loads_a && rank == 0) mbar_arrive_expect_tx(smem_u32(&bars->full[s]), 2 * STAGE_BYTES);
          const uint32_t fb = full_leader0 + static_cast<uint32_t>(s) * 8u;
          if (st < KB) {
            if (loads_a) {
              gemm::tma_load_2d_pair(dst, map_i, fb, st * BK, ca);
            } else {
              gemm::tma_load_2d_pair(dst, map_i, fb, st * BK, cb0);
              gemm::tma_load_2d_pair(dst + HN * BK, map_i, fb, st * BK, cb1);
            }
          } else {
            const int c = st - KB;
            if (loads_a) {
              gemm::tma_load_3d_pair(dst, map_o, fb, 0, ca, c);
            } else {
              gemm::tma_load_3d_pair(dst, map_o, fb, 0, cb0, c);
              gemm::tma_load_3d_pair(dst + HN * BK, map_o, fb, 0, cb1, c);
            }
          }
          ++issued;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok && loads_a && rank == 0) {
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
      // ---------------------------------------------------------------- MMA issuer
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = 0; it < L && ok; ++it) {
        const uint32_t tp = static_cast<uint32_t>(it & 1);
        // the accumulator is free once the previous tile's epilogue released it
        if (!mbar_wait(smem_u32(&bars->tmem_empty), tp ^ 1u, abort_flag, lim)) break;
        tc_fence_after();
        for (int st = 0; st < KB + OC && ok; ++st) {
          if (st == KB) {
            // int8 phase done: the epilogue converts the accumulator, then the outlier
            // MMAs accumulate on top
            gemm::umma_commit_pair(smem_u32(&bars->int_full));
            if (!mbar_wait(smem_u32(&bars->converted), tp, abort_flag, lim)) {
              ok = false;
              break;
            }
            tc_fence_after();
          }
          if (!mbar_wait(smem_u32(&bars->full[s]), ph, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = ring + s * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t d = tmem_base + static_cast<uint32_t>(h * 256);
            const uint32_t sbh = sb + static_cast<uint32_t>(h * HN * BK);
            if (st < KB && kE4M3) {
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk)
                gemm::umma_e4m3_pair(d, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sbh + kk * 32),
                                     IDESC_E4M3, (st | kk) != 0);
            } else if (st < KB) {
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk)
                gemm::umma_i8_pair(d, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sbh + kk * 32),
                                   IDESC_I8, (st | kk) != 0);
            } else {
#pragma unroll
              for (int kk = 0; kk < BK / 32; ++kk)
                gemm::umma_f16_pair(d, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sbh + kk * 32),
                                    IDESC_F16, 1u);
            }
          }
          gemm::umma_commit_pair(smem_u32(&bars->empty[s]));
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        // the tile is final (with outlier columns: after their MMAs; int_full was committed
        // at the end of the int8 phase)
        if (ok) gemm::umma_commit_pair(smem_u32(&bars->tmem_full));
      }
      int no_abort = 0;
      gemm::umma_commit_pair(smem_u32(&bars->drain));
      mbar_wait(smem_u32(&bars->drain), 0u, &no_abort, lim);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------------ epilogue warps
    const int q = warp & 3;
    const int et = threadIdx.x - 64;  // 0..127 among the epilogue threads
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const bool vec_ok = (a.N % 8) == 0;
    bool dead = false;
    int cbuf = 0;
    for (int it = 0; it < L; ++it) {
      const uint32_t tp = static_cast<uint32_t>(it & 1);
      int m0, n0;
      tile_mn(it, m0, n0);
      const int trow0 = m0 + static_cast<int>(rank) * HM + q * 32;
      const int t = trow0 + lane;
      const bool row_ok = t < a.T;
      float* ws = colbuf + (it & 1) * (2 * TN);
      float* bs = ws + TN;
      for (int j = et; j < TN; j += 128) {
        const int n = n0 + j;
        ws[j] = n < a.N ? __ldg(a.SCB + n) * kInvQ : 0.0f;
        bs[j] = (n < a.N && a.bias) ? __half2float(a.bias[n]) : 0.0f;
      }
      gemm::epilogue_bar();
      if (dead) continue;
      const float sx = row_ok ? __ldg(a.SCx + t) * kInvQ : 0.0f;
      if (OC > 0) {
        bool got = mbar_wait(smem_u32(&bars->int_full), tp, abort_flag, lim);
        if (!__all_sync(0xffffffffu, got)) {
          dead = true;
          continue;
        }
        tc_fence_after();
        // two chunks of 32 columns in flight: chunk c + 1 loads while chunk c converts
        auto convert = [&](int c, uint32_t (&r)[32]) {
#pragma unroll
          for (int j = 0; j < 32; ++j) r[j] = __float_as_uint(gemm::acc_value<kE4M3>(r[j]) * sx);
          gemm::tmem_st_32x32b_x32(lane_base + static_cast<uint32_t>(c * 32), r);
        };
        uint32_t ra[32], rb[32];
        tmem_ld_32x32b_x32(lane_base, ra);
#pragma unroll 1
        for (int c = 0; c < TN / 32; c += 2) {
          tmem_ld_wait_regs(ra);
          tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>((c + 1) * 32), rb);
          convert(c, ra);
          tmem_ld_wait_regs(rb);
          if (c + 2 < TN / 32)
            tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>((c + 2) * 32), ra);
          convert(c + 1, rb);
        }
        gemm::tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) gemm::mbar_arrive_remote(gemm::map_to_rank(smem_u32(&bars->converted), 0));
      }
      {
        bool got = mbar_wait(smem_u32(&bars->tmem_full), tp, abort_flag, lim);
        if (!__all_sync(0xffffffffu, got)) {
          dead = true;
          continue;
        }
      }
      tc_fence_after();
      // one chunk of 32 columns: scale, bias, fp16, out through shared memory by TMA
      auto store_chunk = [&](int c, const uint32_t (&r)[32]) {
        const int c0 = n0 + c * 32;
        if (c0 >= a.N || trow0 >= a.T) return;
        float v[32];
        gemm::epilogue_values<kE4M3>(r, OC, sx, ws + c * 32, bs + c * 32, v);
        if (a.c_tma) {
          const uint32_t sb = cstage + static_cast<uint32_t>((q * 2 + cbuf) * 2048);
          if (lane == 0) gemm::bulk_wait_read_1();
          __syncwarp();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            __half2 h0 = __floats2half2_rn(v[8 * q4 + 0], v[8 * q4 + 1]);
            __half2 h1 = __floats2half2_rn(v[8 * q4 + 2], v[8 * q4 + 3]);
            __half2 h2 = __floats2half2_rn(v[8 * q4 + 4], v[8 * q4 + 5]);
            __half2 h3 = __floats2half2_rn(v[8 * q4 + 6], v[8 * q4 + 7]);
            gemm::sts_v4(sb + static_cast<uint32_t>(lane * 64 + q4 * 16),
                         *reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1),
                         *reinterpret_cast<uint32_t*>(&h2), *reinterpret_cast<uint32_t*>(&h3));
          }
          gemm::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            gemm::tma_store_2d(&tmC, sb, c0, trow0);
            gemm::bulk_commit();
          }
          cbuf ^= 1;
        } else if (row_ok) {
          gemm::store_row32_f16(a.C + static_cast<int64_t>(t) * a.N, c0, a.N, v, vec_ok);
        }
      };
      // two chunks in flight: chunk c + 1 loads while chunk c is stored; the accumulator
      // is released as soon as its last chunk is in registers, so the next tile's MMAs
      // start while this tile's last chunk is still being written out
      uint32_t ra[32], rb[32];
      tmem_ld_32x32b_x32(lane_base, ra);
#pragma unroll 1
      for (int c = 0; c < TN / 32; c += 2) {
        tmem_ld_wait_regs(ra);
        tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>((c + 1) * 32), rb);
        store_chunk(c, ra);
        tmem_ld_wait_regs(rb);
        if (c + 2 < TN / 32) {
          tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>((c + 2) * 32), ra);
        } else {
          tc_fence_before();
          __syncwarp();
          if (lane == 0)
            gemm::mbar_arrive_remote(gemm::map_to_rank(smem_u32(&bars->tmem_empty), 0));
        }
        store_chunk(c + 1, rb);
      }
    }
    if (lane == 0) gemm::bulk_wait_all();
  }

  tc_fence_before();
  __syncthreads();
  gemm::cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    gemm::tmem_dealloc_pair(tmem_base, TMEM_COLS);
  }
  gemm::cluster_sync();
}

}  // namespace gemmw
}  // namespace i8

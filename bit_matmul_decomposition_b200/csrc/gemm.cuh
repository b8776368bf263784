// gemm.cuh -- steps 4, 5 and 6 for prefill shapes on the 5th-generation tensor cores.
//
//   acc[t,n]   = sum_k Xq[t,k] * CB[n,k]              tcgen05.mma kind::i8 -> int32 in TMEM
//   acc_o[t,n] = sum_j X_o[t,j] * CB_o[n,j]            tcgen05.mma kind::f16 -> fp32 in TMEM
//   C[t,n]     = fp16((acc * SCx[t]/127 + acc_o) * SCB[n]/127 + bias[n])   (epilogue)
//
// Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at
// scale" (Hugging Face blog), "内部的 MatMul": the int8 product of row-quantised hidden
// states and column-quantised weights, dequantised and added to the fp16 product of the
// outlier columns; "absmax 量化": dequantisation by the outer product of the absmax
// vectors; "用法": the fp16 weights of the outlier product are CB * SCB / 127.
//
// Design (sm_100a, one CTA per SM, persistent over 128 x 256 output tiles):
//   warp 0      TMA producer: Xq/CB tiles (128 B of K per stage, 128-byte swizzle), then
//               the X_o/CB_o outlier chunks (64 fp16 per stage), into a 4-stage ring.
//   warp 1      TMEM allocator and MMA issuer (one thread): 4 MMAs of K=32 bytes per
//               stage; commits free the ring slot and, per tile, hand the accumulator
//               to the epilogue.
//   warps 2..5  epilogue: tcgen05.ld of 32 columns at a time, the fp32 dequant / outlier
//               add / bias, fp16 stores.  Warp w reads TMEM lanes 32*(w%4)..+31.
// TMEM (512 columns): with no outliers, two int32 accumulators of 256 columns alternate
// so the epilogue of tile i overlaps the MMAs of tile i+1; with outliers, one int32
// accumulator [0,256) and one fp32 outlier accumulator [256,512).
#pragma once

#include "common.cuh"

namespace i8 {
namespace gemm {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;  // bytes of K per stage
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK;
constexpr int B_BYTES = BN * BK;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 192;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t IDESC_I8 = idesc_s8_s32(BM, BN);
constexpr uint32_t IDESC_F16 = idesc_f16_f32(BM, BN);
constexpr int BAR_BYTES = 256;
constexpr size_t SMEM_BYTES = static_cast<size_t>(STAGES) * STAGE_BYTES + BAR_BYTES + 1024;

static_assert(BM == 128 && BN % 16 == 0 && BN <= 256, "UMMA M=128 shape");
static_assert(THREADS == 192, "warp roles assume 6 warps");

struct Args {
  int T, N, K;
  int m_tiles, n_tiles, k_blocks;
  const int32_t* n_outliers;  // device scalar, NULL = no outlier phase
  const float* SCx;
  const float* SCB;
  const __half* bias;  // nullable
  __half* C;
  int32_t* acc_out;  // raw-accumulator mode
  uint64_t wait_limit_ns;
};

struct SmemBars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(SmemBars) <= BAR_BYTES, "barrier block");

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

template <bool kRaw>
__global__ void __launch_bounds__(THREADS, 1)
    i8_gemm_tcgen05_kernel(const __grid_constant__ CUtensorMap tmA,
                           const __grid_constant__ CUtensorMap tmB,
                           const __grid_constant__ CUtensorMap tmAo,
                           const __grid_constant__ CUtensorMap tmBo, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t ring = raw_s + pad;  // 1024-aligned shared address of stage 0
  SmemBars* bars = reinterpret_cast<SmemBars*>(smem + static_cast<size_t>(STAGES) * STAGE_BYTES);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->tmem_full[b]), 1);
      mbar_init(smem_u32(&bars->tmem_empty[b]), 128);
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
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_base), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_base;

  const int n_o = (a.n_outliers != nullptr) ? max(0, __ldg(a.n_outliers)) : 0;
  const int o_chunks = (n_o + 63) >> 6;
  const int nbuf = (o_chunks == 0) ? 2 : 1;
  const int num_tiles = a.m_tiles * a.n_tiles;
  const int steps_per_tile = a.k_blocks + o_chunks;
  const uint64_t lim = a.wait_limit_ns;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ TMA producer
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % a.m_tiles) * BM;
        const int n0 = (tile / a.m_tiles) * BN;
        for (int kb = 0; kb < steps_per_tile; ++kb) {
          if (!mbar_wait(smem_u32(&bars->empty[s]), ph ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          const uint32_t sa = ring + s * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          const uint32_t fb = smem_u32(&bars->full[s]);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          if (kb < a.k_blocks) {
            tma_load_2d(sa, &tmA, fb, kb * BK, m0);
            tma_load_2d(sb, &tmB, fb, kb * BK, n0);
          } else {
            const int c = kb - a.k_blocks;
            tma_load_3d(sa, &tmAo, fb, 0, m0, c);
            tma_load_3d(sb, &tmBo, fb, 0, n0, c);
          }
          ++issued;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
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
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int it = 0;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++it) {
        const int b = (nbuf == 2) ? (it & 1) : 0;
        const uint32_t use = (nbuf == 2) ? static_cast<uint32_t>(it >> 1) : static_cast<uint32_t>(it);
        if (!mbar_wait(smem_u32(&bars->tmem_empty[b]), (use & 1u) ^ 1u, abort_flag, lim)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_int = tmem_base + static_cast<uint32_t>(b * BN);
        const uint32_t d_out = tmem_base + static_cast<uint32_t>(BN);
        for (int kb = 0; kb < steps_per_tile; ++kb) {
          if (!mbar_wait(smem_u32(&bars->full[s]), ph, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = ring + s * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
          if (kb < a.k_blocks) {
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              umma_i8(d_int, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32), IDESC_I8,
                      (kb | kk) != 0);
          } else {
            const int c = kb - a.k_blocks;
#pragma unroll
            for (int kk = 0; kk < BK / 32; ++kk)
              umma_f16(d_out, sdesc_k_sw128(sa + kk * 32), sdesc_k_sw128(sb + kk * 32),
                       IDESC_F16, (c | kk) != 0);
          }
          umma_commit(smem_u32(&bars->empty[s]));
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(smem_u32(&bars->tmem_full[b]));
      }
      // every MMA issued by this thread completes before TMEM is released
      int no_abort = 0;
      umma_commit(smem_u32(&bars->drain));
      mbar_wait(smem_u32(&bars->drain), 0u, &no_abort, lim);
    }
  } else {
    // -------------------------------------------------------------- epilogue warps
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    const bool vec_ok = (a.N % 8) == 0;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const int b = (nbuf == 2) ? (it & 1) : 0;
      const uint32_t use = (nbuf == 2) ? static_cast<uint32_t>(it >> 1) : static_cast<uint32_t>(it);
      // all 32 lanes must take the same branch: tcgen05.ld below is warp-collective
      const bool got = mbar_wait(smem_u32(&bars->tmem_full[b]), use & 1u, abort_flag, lim);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int m0 = (tile % a.m_tiles) * BM;
      const int n0 = (tile / a.m_tiles) * BN;
      const int t = m0 + row;
      const bool row_ok = t < a.T;
      float sx = 0.0f;
      if (!kRaw && row_ok) sx = __ldg(a.SCx + t) * (1.0f / 127.0f);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        uint32_t o[32];
        tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(b * BN + c * 32), r);
        if (!kRaw && nbuf == 1) tmem_ld_32x32b_x32(lane_base + static_cast<uint32_t>(BN + c * 32), o);
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
          } else {
            float v[32];
#pragma unroll
            for (int j = 0; j < 32; ++j) {
              const int n = min(c0 + j, a.N - 1);
              const float ws = __ldg(a.SCB + n) * (1.0f / 127.0f);
              const float bn = a.bias ? __half2float(a.bias[n]) : 0.0f;
              const float oj = (nbuf == 1) ? __uint_as_float(o[j]) : 0.0f;
              const float part = fmaf(static_cast<float>(static_cast<int32_t>(r[j])), sx, oj);
              v[j] = fmaf(part, ws, bn);
            }
            store_row32_f16(a.C + static_cast<int64_t>(t) * a.N, c0, a.N, v, vec_ok);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(smem_u32(&bars->tmem_empty[b]));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace gemm
}  // namespace i8

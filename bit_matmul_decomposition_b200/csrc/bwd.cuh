// bwd.cuh -- the backward of the layer's fp16-weight training mode, on the 5th-generation
// tensor cores, and the small HBM-bound passes around it:
//
//   dX[T,K] = dY[T,N] * W[N,K]            f16_gemm_kernel<false, true>   (A K-major, B MN-major)
//   dW[N,K] = dY[T,N]^T * X[T,K]          f16_gemm_kernel<true,  true>   (A MN-major, B MN-major)
//   db[N]   = sum_t dY[t,N]               bias_grad_kernel
//   W'[N,K] = CB[N,K] * SCB[N] / 127      dequantize_kernel (the weight the int8 forward uses;
//                                         e4m3 codes: their values * SCB / 448)
//
// Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at scale"
// (Hugging Face blog), "用法": has_fp16_weights=True keeps fp16 weights for int8/fp16
// mixed-precision training, and CB * SCB / 127 recovers the weight.  The blog gives no
// gradient formulas; the plainest reading is the backward of y = x W^T + b passed straight
// through the quantisation, which these kernels compute.
//
// f16_gemm_kernel computes C[m,n] = sum_r A(m,r) * B(n,r) with fp16 operands, fp32
// accumulation in TMEM and an fp16 output.  An operand is K-major when its rows run along
// the reduction (A(m,r) at A[m * ld + r]) and MN-major when they run along m or n
// (A(m,r) at A[r * ld + m]); the instruction descriptor's transpose bits tell the tensor
// cores which.  Design as the forward GEMM (gemm.cuh): persistent clusters of two CTAs,
// tcgen05.mma.cta_group::2 kind::f16 with 256 x 256 output tiles, a 6-stage TMA ring of
// 64 reduction elements (128 B) per stage, TMA without multicast, two 256-column TMEM
// accumulators so that a tile's epilogue overlaps the next tile's MMAs.  Warps: 0 loads A
// and arms the leader's barrier, 6 loads B, 1 allocates TMEM and (leader lane 0) issues
// the MMAs, 2..5 drain TMEM into fp16 and store C by TMA.
// Shared-memory operand layouts (128-byte swizzle, as TMA writes them):
//   K-major:  one box of 128 rows x 64 elements; rows of 128 B, 8-row atoms of 1024 B.
//             Descriptor: SBO = 1024 B (next 8 rows); K steps of 16 advance the start 32 B.
//   MN-major: two boxes of 64 reduction rows x 64 elements (m or n), 8 KB each, the second
//             holding elements 64..127.  Descriptor: LBO = 8192 B (next 64 elements of m or
//             n), SBO = 1024 B (next 8 reduction rows); K steps of 16 advance the start by
//             16 rows = 2048 B.
#pragma once

#include "common.cuh"
#include "gemm.cuh"
#include "quant.cuh"

namespace i8 {
namespace bwd {

using gemm::TM;
using gemm::TN;
using gemm::HM;
using gemm::HN;
constexpr int BK = 64;                       // reduction elements per stage (128 B)
constexpr int STAGES = 6;
constexpr int A_BYTES = HM * BK * 2;         // 16 KB per CTA
constexpr int B_BYTES = HN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int THREADS = 224;
constexpr uint32_t TMEM_COLS = 512;
constexpr int GROUP_M = 16;
constexpr int CST_BYTES = 4 * 2 * 32 * 64;   // fp16 C staging: per epilogue warp two 32x32 blocks
constexpr int BAR_BYTES = 256;
constexpr size_t SMEM_BYTES =
    static_cast<size_t>(STAGES) * STAGE_BYTES + CST_BYTES + BAR_BYTES + 1024;
static_assert(SMEM_BYTES <= 232448, "shared memory per CTA");

// fp16 x fp16 -> fp32 instruction descriptor, M = 256, N = 256, with the transpose bits
// (bit 15: A MN-major, bit 16: B MN-major)
template <bool kAMN, bool kBMN>
__host__ __device__ constexpr uint32_t idesc() {
  return idesc_f16_f32(TM, TN) | (kAMN ? (1u << 15) : 0u) | (kBMN ? (1u << 16) : 0u);
}

// Shared-memory descriptor of an MN-major operand in the 128-byte-swizzle layout above:
//   bits 0-13 start >> 4, 16-29 LBO >> 4 (8192 B), 32-45 SBO >> 4 (1024 B),
//   46-47 version 1, 61-63 swizzle mode 2 (128 B).
__device__ __forceinline__ uint64_t sdesc_mn_sw128(uint32_t smem_addr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((smem_addr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(8192u >> 4) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

struct Args {
  int M, Nc, R;                  // C is [M, Nc]; the reduction has R terms
  int m_tiles, n_tiles, k_blocks;
  __half* C;                     // written by threads when !c_tma
  int ldc;
  bool c_tma;
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

template <bool kAMN, bool kBMN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    f16_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const Args a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* smem = smem_raw + pad;
  const uint32_t ring = raw_s + pad;
  const uint32_t cstage = ring + static_cast<uint32_t>(STAGES * STAGE_BYTES);
  SmemBars* bars =
      reinterpret_cast<SmemBars*>(smem + static_cast<size_t>(STAGES) * STAGE_BYTES + CST_BYTES);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = gemm::cluster_rank();
  volatile int* abort_flag = &bars->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&bars->full[s]), 1);
      mbar_init(smem_u32(&bars->empty[s]), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(smem_u32(&bars->tmem_full[b]), 1);
      mbar_init(smem_u32(&bars->tmem_empty[b]), 8);   // 4 epilogue warps x 2 CTAs
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
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
  grid_dep_wait();

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
      const bool loads_a = (warp == 0);
      const bool mn = loads_a ? kAMN : kBMN;
      const CUtensorMap* map = loads_a ? &tmA : &tmB;
      const uint32_t half_off = loads_a ? 0u : static_cast<uint32_t>(A_BYTES);
      const uint32_t full_leader0 = gemm::map_to_rank(smem_u32(&bars->full[0]), 0);
      int s = 0;
      uint32_t ph = 0, issued = 0;
      bool ok = true;
      for (int it = 0; it < L && ok; ++it) {
        int m0, n0;
        tile_mn(it, m0, n0);
        const int c0 = (loads_a ? m0 + static_cast<int>(rank) * HM : n0 + static_cast<int>(rank) * HN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(smem_u32(&bars->empty[s]), ph ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          const uint32_t dst = ring + s * STAGE_BYTES + half_off;
          if (loads_a && rank == 0)
            mbar_arrive_expect_tx(smem_u32(&bars->full[s]), 2 * STAGE_BYTES);
          const uint32_t fb = full_leader0 + static_cast<uint32_t>(s) * 8u;
          if (mn) {
            gemm::tma_load_2d_pair(dst, map, fb, c0, kb * BK);
            gemm::tma_load_2d_pair(dst + 8192u, map, fb, c0 + 64, kb * BK);
          } else {
            gemm::tma_load_2d_pair(dst, map, fb, kb * BK, c0);
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
      constexpr uint32_t ID = idesc<kAMN, kBMN>();
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = 0; it < L && ok; ++it) {
        const int b = it & 1;
        const uint32_t use = static_cast<uint32_t>(it >> 1);
        if (!mbar_wait(smem_u32(&bars->tmem_empty[b]), (use & 1u) ^ 1u, abort_flag, lim)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + static_cast<uint32_t>(b * TN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!mbar_wait(smem_u32(&bars->full[s]), ph, abort_flag, lim)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = ring + s * STAGE_BYTES;
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = kAMN ? sdesc_mn_sw128(sa + kk * 2048) : sdesc_k_sw128(sa + kk * 32);
            const uint64_t bd = kBMN ? sdesc_mn_sw128(sb + kk * 2048) : sdesc_k_sw128(sb + kk * 32);
            gemm::umma_f16_pair(d, ad, bd, ID, (kb | kk) != 0);
          }
          gemm::umma_commit_pair(smem_u32(&bars->empty[s]));
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (ok) gemm::umma_commit_pair(smem_u32(&bars->tmem_full[b]));
      }
      int no_abort = 0;
      gemm::umma_commit_pair(smem_u32(&bars->drain));
      mbar_wait(smem_u32(&bars->drain), 0u, &no_abort, lim);
    }
  } else if (warp >= 2 && warp <= 5) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_base = tmem_base + (static_cast<uint32_t>(q * 32) << 16);
    int cbuf = 0;
    for (int it = 0; it < L; ++it) {
      const int b = it & 1;
      const uint32_t use = static_cast<uint32_t>(it >> 1);
      int m0, n0;
      tile_mn(it, m0, n0);
      const int trow0 = m0 + static_cast<int>(rank) * HM + q * 32;
      const int t = trow0 + lane;
      const bool got = mbar_wait(smem_u32(&bars->tmem_full[b]), use & 1u, abort_flag, lim);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const uint32_t tb = lane_base + static_cast<uint32_t>(b * TN);
#pragma unroll 1
      for (int c = 0; c < TN / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tb + static_cast<uint32_t>(c * 32), r);
        tmem_ld_wait();
        const int c0 = n0 + c * 32;
        if (c0 >= a.Nc || trow0 >= a.M) continue;
        if (a.c_tma) {
          const uint32_t sb = cstage + static_cast<uint32_t>((q * 2 + cbuf) * 2048);
          if (lane == 0) gemm::bulk_wait_read_1();
          __syncwarp();
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            __half2 h0 = __floats2half2_rn(__uint_as_float(r[8 * q4 + 0]), __uint_as_float(r[8 * q4 + 1]));
            __half2 h1 = __floats2half2_rn(__uint_as_float(r[8 * q4 + 2]), __uint_as_float(r[8 * q4 + 3]));
            __half2 h2 = __floats2half2_rn(__uint_as_float(r[8 * q4 + 4]), __uint_as_float(r[8 * q4 + 5]));
            __half2 h3 = __floats2half2_rn(__uint_as_float(r[8 * q4 + 6]), __uint_as_float(r[8 * q4 + 7]));
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
        } else if (t < a.M) {
          __half* crow = a.C + static_cast<int64_t>(t) * a.ldc;
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c0 + j < a.Nc) crow[c0 + j] = __float2half_rn(__uint_as_float(r[j]));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) gemm::mbar_arrive_remote(gemm::map_to_rank(smem_u32(&bars->tmem_empty[b]), 0));
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

// ------------------------------------------------------------------ bias gradient
// db[n] = fp16(sum_t dY[t,n]), summed in fp32 in a fixed order (deterministic): a CTA owns
// 64 columns (a lane two of them, so a warp reads 128 contiguous bytes of a row); its 8
// warps take every 8th row, then the 8 partial sums are added in warp order.
constexpr int kBiasThreads = 256;

__global__ void __launch_bounds__(kBiasThreads)
    bias_grad_kernel(const __half* __restrict__ dY, int64_t T, int64_t N, __half* __restrict__ db) {
  __shared__ float2 part[kBiasThreads / 32][32];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t n = static_cast<int64_t>(blockIdx.x) * 64 + 2 * lane;
  float2 acc = make_float2(0.0f, 0.0f);
  if (n < N) {
    const bool pair = n + 1 < N;
    int64_t t = warp;
    for (; t + 3 * 8 < T; t += 4 * 8) {   // four rows' loads in flight
      float2 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const __half* p = dY + (t + u * 8) * N + n;
        v[u] = pair ? __half22float2(*reinterpret_cast<const __half2*>(p))
                    : make_float2(__half2float(*p), 0.0f);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        acc.x += v[u].x;
        acc.y += v[u].y;
      }
    }
    for (; t < T; t += 8) {
      const __half* p = dY + t * N + n;
      const float2 v = pair ? __half22float2(*reinterpret_cast<const __half2*>(p))
                            : make_float2(__half2float(*p), 0.0f);
      acc.x += v.x;
      acc.y += v.y;
    }
  }
  part[warp][lane] = acc;
  __syncthreads();
  if (warp == 0 && n < N) {
    float2 s = part[0][lane];
    for (int w = 1; w < kBiasThreads / 32; ++w) {
      s.x += part[w][lane].x;
      s.y += part[w][lane].y;
    }
    db[n] = __float2half_rn(s.x);
    if (n + 1 < N) db[n + 1] = __float2half_rn(s.y);
  }
}

// ------------------------------------------------------------------ dequantised weight
// W'[n,k] = fp16(code(CB[n,k]) * fl32(SCB[n] / 127)), or with e4m3 codes their values times
// fl32(SCB[n] / 448).  A grid-stride loop over 16-byte groups of codes (16 per thread and
// step), one 32-byte store of fp16 per group.
constexpr int kDequantThreads = 256;

__global__ void __launch_bounds__(kDequantThreads)
    dequantize_kernel(const int8_t* __restrict__ CB, const float* __restrict__ SCB, int64_t N,
                      int64_t K, __half* __restrict__ W, bool e4m3) {
  const int64_t groups = N * K / 16;     // K % 16 == 0: a group never crosses a row
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * kDequantThreads + threadIdx.x; g < groups;
       g += static_cast<int64_t>(gridDim.x) * kDequantThreads) {
    const int64_t n = (g * 16) / K;
    const float s = __fdiv_rn(__ldg(SCB + n), e4m3 ? 448.0f : 127.0f);
    const uint4 c = ldg_v4(CB + g * 16);
    const uint32_t w[4] = {c.x, c.y, c.z, c.w};
    uint32_t o[8];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t b0 = (w[i] >> (16 * h)) & 0xffu, b1 = (w[i] >> (16 * h + 8)) & 0xffu;
        float v0, v1;
        if (e4m3) {
          v0 = __half2float(code_to_half(static_cast<int>(b0), true));
          v1 = __half2float(code_to_half(static_cast<int>(b1), true));
        } else {
          v0 = static_cast<float>(static_cast<int8_t>(b0));
          v1 = static_cast<float>(static_cast<int8_t>(b1));
        }
        __half2 hv = __floats2half2_rn(v0 * s, v1 * s);
        o[2 * i + h] = *reinterpret_cast<uint32_t*>(&hv);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(W + g * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

}  // namespace bwd
}  // namespace i8

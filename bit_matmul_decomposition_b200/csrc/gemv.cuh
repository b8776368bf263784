// gemv.cuh -- steps 4, 5 and 6 for decode batches (T <= 16), where the layer is a stream
// of CB through HBM: each CB byte is used by at most 16 tokens, so the bound is memory,
// not the tensor pipe.  gemv_stream_kernel computes the int8 K-slice partial sums;
// gemv_finalize_kernel adds them up and applies the fp16 outlier product, the
// dequantisation and the bias.
//
// Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at
// scale" (Hugging Face blog), "内部的 MatMul" (int8 product, dequantisation, fp16
// outlier product); "改进范围" notes that small-batch inference was the slow case.
//
// K-slicing keeps the Xq slice resident in shared memory while a CTA streams many 16-row
// tiles of CB.  Within one 64-byte step a thread takes 16 contiguous CB bytes of rows g
// and g+8 and the 16 matching Xq bytes of token g; two m16n8k32 MMAs consume them.  The
// k order inside the step is permuted identically for A and B, which leaves each dot
// product unchanged.
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace i8 {
namespace gemv {

constexpr int WARPS = 8;             // slice lengths are whole multiples of WARPS * 64 bytes
constexpr int ROWS = 16;          // CB rows per tile (MMA M)
constexpr int SLICE_TARGET = 3584;  // bytes of K per slice (before rounding)

__host__ __device__ inline int64_t slice_bytes(int64_t K) {
  // rounded to WARPS * 64 so that every warp owns a whole number of 64-byte steps
  const int64_t S = (K + SLICE_TARGET - 1) / SLICE_TARGET;
  const int64_t per = (K + S - 1) / S;
  return ((per + WARPS * 64 - 1) / (WARPS * 64)) * (WARPS * 64);
}

__host__ __device__ inline int64_t num_slices(int64_t K) {
  const int64_t ks = slice_bytes(K);
  return (K + ks - 1) / ks;
}


__device__ __forceinline__ void mma_s8_16816(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Decode kernels (steps 4, 5 and 6 for T <= 16), two launches after the fused prepare.
//
// gemv_stream_kernel: warp CW (one thread) streams CB through a ring of STAGES stages,
// each 16 rows x CH bytes of K, loaded as 2-D TMA boxes of 256 B x 16 rows (no swizzle:
// the widest box TMA takes, which streams HBM best -- ~6 TB/s measured on B200 for this
// layout).  The CW compute warps each own one 64-byte MMA step of every stage and
// accumulate, over the tile's stages of their CTA's K-slice,
//   P[slice][t][n] = sum_{k in slice} Xq[t,k] * CB[n,k]     (int32, mma.sync m16n8k32)
// in registers; at the tile's end the warps' partials are reduced in a fixed order.
// The loop carries nothing but the int8 product: the outlier columns are a handful, and
// any per-column work inside it lands on the same warp in every tile and holds up the
// tile-end barrier.
//
// gemv_finalize_kernel: one thread per output channel n and group of TG tokens sums the
// slice partials (exact int32) and gathers the n_o outlier bytes CB[n, idx[j]] once,
// applying each to the group's tokens (fp32), then writes
//   C[t,n] = fp16((P[t,n] * SCx[t]/127 + sum_j X_o[t,j] * CB[n,idx[j]]) * SCB[n]/127 + bias[n]).
constexpr int BOXW = 256;                   // bytes of K per TMA box
constexpr int CW = 8;                       // compute warps, one 64-byte step each
constexpr int STREAM_THREADS = (CW + 1) * 32;
constexpr int CH = 64 * CW;                 // bytes of K per stage per row
constexpr int BOXES = CH / BOXW;            // TMA boxes per stage
constexpr int STAGES = 16;
constexpr int STAGE_BYTES = ROWS * CH;      // 8 KB
constexpr int RP = ROWS + 4;                // row pitch of the reduction buffer (in words):
                                            // fragment stores and the row-fastest reads
                                            // then fall on (nearly) distinct banks
constexpr int TG = 4;                       // tokens per finalize thread
constexpr int FIN_THREADS = 128;

static_assert(CH % BOXW == 0, "whole boxes per stage");
static_assert(SLICE_TARGET % CH == 0 && (WARPS * 64) % CH == 0, "slices hold whole stages");

__host__ inline size_t stream_smem_bytes(int nt, int64_t K) {
  return 1024 + static_cast<size_t>(STAGES) * STAGE_BYTES +
         static_cast<size_t>(nt * 8) * static_cast<size_t>(slice_bytes(K) + 16) +
         static_cast<size_t>(CW) * RP * nt * 8 * 4 + 2 * STAGES * 8;
}

template <int NT>
__global__ void __launch_bounds__(STREAM_THREADS, 1)
    gemv_stream_kernel(const __grid_constant__ CUtensorMap tmCB, const int8_t* __restrict__ Xq,
                       int T, int64_t N, int64_t K, int32_t* __restrict__ P, uint64_t lim) {
  extern __shared__ uint8_t smraw[];
  const uint32_t raw_s = smem_u32(smraw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* sm = smraw + pad;
  const uint32_t ring = raw_s + pad;
  const int64_t KS = slice_bytes(K);
  const int S = static_cast<int>(num_slices(K));
  const int64_t pitch = KS + 16;
  uint8_t* xs = sm + static_cast<size_t>(STAGES) * STAGE_BYTES;
  int32_t* red = reinterpret_cast<int32_t*>(xs + NT * 8 * pitch);
  uint64_t* full = reinterpret_cast<uint64_t*>(red + CW * RP * NT * 8);
  uint64_t* empty = full + STAGES;
  __shared__ int s_abort;

  const int slice = blockIdx.x % S;
  const int cta_in_slice = blockIdx.x / S;
  const int ctas_in_slice = (static_cast<int>(gridDim.x) - slice + S - 1) / S;
  const int64_t k0 = static_cast<int64_t>(slice) * KS;
  const int64_t klen = min(KS, K - k0);
  const int spt = static_cast<int>((klen + CH - 1) / CH);   // stages per tile
  const int64_t n_tiles = (N + ROWS - 1) / ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), CW);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == CW && lane == 0) tma_prefetch_desc(&tmCB);
  grid_dep_wait();    // Xq comes from the previous kernel
  grid_dep_launch();  // the finalize kernel may start launching
  // stage Xq[:, k0 : k0+KS] (tokens >= T and columns >= K are zero)
  const int64_t vec_per_row = KS / 16;
  for (int64_t i = threadIdx.x; i < NT * 8 * vec_per_row; i += STREAM_THREADS) {
    const int tok = static_cast<int>(i / vec_per_row);
    const int64_t c16 = i - tok * vec_per_row;
    const int64_t k = k0 + c16 * 16;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (tok < T && k < K) v = ldg_v4(Xq + static_cast<int64_t>(tok) * K + k);
    *reinterpret_cast<uint4*>(xs + tok * pitch + c16 * 16) = v;
  }
  __syncthreads();
  volatile int* abort_flag = &s_abort;

  if (warp == CW) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      bool ok = true;
      for (int64_t tile = cta_in_slice; tile < n_tiles && ok; tile += ctas_in_slice) {
        const int y = static_cast<int>(tile * ROWS);
        for (int st = 0; st < spt; ++st) {
          if (!mbar_wait(smem_u32(empty + s), ph ^ 1u, abort_flag, lim)) {
            ok = false;
            break;
          }
          const uint32_t fb = smem_u32(full + s);
          mbar_arrive_expect_tx(fb, STAGE_BYTES);
          const int x = static_cast<int>(k0 + static_cast<int64_t>(st) * CH);
#pragma unroll
          for (int c = 0; c < BOXES; ++c)
            tma_load_2d(ring + s * STAGE_BYTES + c * (ROWS * BOXW), &tmCB, fb, x + c * BOXW, y);
          ++issued;
          if (++s == STAGES) {
            s = 0;
            ph ^= 1u;
          }
        }
      }
      if (!ok) {
        // wind down: let the copies in flight land (bounded) before the CTA exits
        int no_abort = 0;
        const uint32_t inflight = issued < STAGES ? issued : STAGES;
        for (uint32_t i = 0; i < inflight; ++i) {
          const uint32_t u = issued - 1 - i;
          mbar_wait(smem_u32(full + u % STAGES), (u / STAGES) & 1u, &no_abort, lim);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ compute warps
    const int g = lane >> 2, q = lane & 3;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int64_t tile = cta_in_slice; tile < n_tiles; tile += ctas_in_slice) {
      int c[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0;
      for (int st = 0; st < spt; ++st) {
        if (ok) {
          const bool got = mbar_wait(smem_u32(full + s), ph, abort_flag, lim);
          ok = __all_sync(0xffffffffu, got);
        }
        if (ok) {
          // this warp's 64-byte step of the stage: box warp / 4, bytes 64 * (warp % 4) of
          // each 256-byte row; k offset within the slice = stage * CH + 64 * warp
          const uint32_t rowbase = ring + s * STAGE_BYTES + (warp >> 2) * (ROWS * BOXW) +
                                   (warp & 3) * 64 + q * 16;
          const int64_t kx = static_cast<int64_t>(st) * CH + 64 * warp + 16 * q;
          const uint4 A0 = lds_v4(rowbase + g * BOXW);
          const uint4 A1 = lds_v4(rowbase + (g + 8) * BOXW);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint4 B = *reinterpret_cast<const uint4*>(xs + (nt * 8 + g) * pitch + kx);
            mma_s8_16816(c[nt], A0.x, A1.x, A0.y, A1.y, B.x, B.y);
            mma_s8_16816(c[nt], A0.z, A1.z, A0.w, A1.w, B.z, B.w);
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(empty + s));
        }
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      }
      // ---- reduce the warps' partials of this tile (fixed order) and write P;
      // the buffer is [warp][token][row] with row pitch RP
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int i0 = (warp * (NT * 8) + nt * 8 + 2 * q) * RP + g;
        red[i0] = c[nt][0];
        red[i0 + RP] = c[nt][1];
        red[i0 + 8] = c[nt][2];
        red[i0 + RP + 8] = c[nt][3];
      }
      asm volatile("bar.sync 1, %0;" ::"n"(CW * 32) : "memory");
      const int64_t n0 = tile * ROWS;
      for (int i = threadIdx.x; i < ROWS * NT * 8; i += CW * 32) {
        const int tok = i / ROWS, rr = i - tok * ROWS;   // consecutive threads: consecutive n
        int32_t sum = 0;
#pragma unroll
        for (int w = 0; w < CW; ++w) sum += red[(w * (NT * 8) + tok) * RP + rr];
        const int64_t n = n0 + rr;
        if (tok < T && n < N) P[(static_cast<int64_t>(slice) * T + tok) * N + n] = sum;
      }
      asm volatile("bar.sync 1, %0;" ::"n"(CW * 32) : "memory");
    }
  }
  __syncthreads();
}

// One thread per output channel n (consecutive threads on consecutive n) and group of TG
// tokens (grid.y): the outlier bytes CB[n, idx[j]] are gathered once per group (8 loads in
// flight; later groups find them in L2) and applied to the group's tokens in fp32, column
// order j = 0 .. n_o-1; the slice partials are summed exactly (int32, slice order).
// kRaw writes the int32 sums.
template <bool kRaw>
__global__ void __launch_bounds__(FIN_THREADS)
    gemv_finalize_kernel(const int32_t* __restrict__ P, int S, int T, int64_t N, int64_t K,
                         const float* __restrict__ SCx, const float* __restrict__ SCB,
                         const __half* __restrict__ bias, const int8_t* __restrict__ CB,
                         const int32_t* __restrict__ idx, const int32_t* __restrict__ n_o_ptr,
                         const __half* __restrict__ X_o, __half* __restrict__ C,
                         int32_t* __restrict__ acc_out) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int t0 = blockIdx.y * TG;
  const int tn = min(TG, T - t0);
  grid_dep_wait();    // the partial sums come from the previous kernel
  if (n >= N) return;
  int32_t acc[TG];
#pragma unroll
  for (int u = 0; u < TG; ++u) acc[u] = 0;
  for (int sl = 0; sl < S; ++sl) {
    const int32_t* p = P + (static_cast<int64_t>(sl) * T + t0) * N + n;
#pragma unroll
    for (int u = 0; u < TG; ++u)
      if (u < tn) acc[u] += __ldcs(p + u * N);
  }
  if (kRaw) {
#pragma unroll
    for (int u = 0; u < TG; ++u)
      if (u < tn) acc_out[static_cast<int64_t>(t0 + u) * N + n] = acc[u];
    return;
  }
  float o[TG];
#pragma unroll
  for (int u = 0; u < TG; ++u) o[u] = 0.0f;
  const int n_o = n_o_ptr == nullptr ? 0 : __ldg(n_o_ptr);
  const int8_t* cbrow = CB + n * K;
  for (int j0 = 0; j0 < n_o; j0 += 8) {
    float cb[8];
#pragma unroll
    for (int v = 0; v < 8; ++v)
      cb[v] = j0 + v < n_o ? static_cast<float>(cbrow[__ldg(idx + j0 + v)]) : 0.0f;
#pragma unroll
    for (int v = 0; v < 8; ++v) {
      const int j = j0 + v;
      if (j >= n_o) break;
      const __half* xo = X_o + (static_cast<int64_t>(j >> 6) * T + t0) * 64 + (j & 63);
#pragma unroll
      for (int u = 0; u < TG; ++u)
        if (u < tn) o[u] = fmaf(__half2float(xo[u * 64]), cb[v], o[u]);
    }
  }
  const float ws = __ldg(SCB + n) * (1.0f / 127.0f);
  const float bn = bias ? __half2float(bias[n]) : 0.0f;
#pragma unroll
  for (int u = 0; u < TG; ++u) {
    if (u < tn) {
      const float part =
          fmaf(static_cast<float>(acc[u]), __ldg(SCx + t0 + u) * (1.0f / 127.0f), o[u]);
      C[static_cast<int64_t>(t0 + u) * N + n] = __float2half_rn(fmaf(part, ws, bn));
    }
  }
}

}  // namespace gemv
}  // namespace i8

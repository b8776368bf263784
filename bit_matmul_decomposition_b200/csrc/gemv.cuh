// gemv.cuh -- steps 4, 5 and 6 for decode batches (T <= 16), where the layer is a stream
// of CB through HBM: each CB byte is used by at most 16 tokens, so the bound is memory,
// not the tensor pipe.
//
//   gemv_partial_kernel   int8 x int8 -> int32 partial sums over one K-slice, with the
//                         warp-level tensor-core MMA m16n8k32 (16 CB rows x 8 tokens):
//                         CB streams from HBM in 16-byte loads (no L1 allocation),
//                         the slice of Xq sits in shared memory.
//   gemv_finalize_kernel  sums the K-slice partials (exact int32), then the same
//                         epilogue as the GEMM: (acc*SCx/127 + sum_j X_o*CB_o)*SCB/127 + bias.
//
// Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at
// scale" (Hugging Face blog), "内部的 MatMul" (int8 product, dequantisation, fp16
// outlier product); "改进范围" notes that small-batch inference was the slow case.
//
// K-slicing keeps the Xq slice resident in shared memory while the CTA streams many
// 16-row tiles of CB; partial sums are written once each (no atomics), so the result is
// deterministic.  Within one 64-byte step a thread loads 16 contiguous CB bytes of rows
// g and g+8 and the 16 matching Xq bytes of token g; two MMAs consume them.  The k
// order inside the step is permuted identically for A and B, which leaves each dot
// product unchanged.
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace i8 {
namespace gemv {

constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
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

__host__ inline size_t smem_bytes(int nt, int64_t K) {
  return static_cast<size_t>(nt * 8) * static_cast<size_t>(slice_bytes(K) + 16) +
         static_cast<size_t>(WARPS) * ROWS * nt * 8 * sizeof(int32_t);
}

__device__ __forceinline__ void mma_s8_16816(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// P[slice][t][n] = sum over k in the slice of Xq[t,k] * CB[n,k]   (t < T only)
template <int NT>
__global__ void __launch_bounds__(THREADS)
    gemv_partial_kernel(const int8_t* __restrict__ Xq, const int8_t* __restrict__ CB, int T,
                        int64_t N, int64_t K, int32_t* __restrict__ P) {
  extern __shared__ __align__(16) uint8_t sm[];
  const int64_t KS = slice_bytes(K);
  const int S = static_cast<int>(num_slices(K));
  const int64_t pitch = KS + 16;
  const int slice = blockIdx.x % S;
  const int cta_in_slice = blockIdx.x / S;
  const int ctas_in_slice = (static_cast<int>(gridDim.x) - slice + S - 1) / S;
  const int64_t k0 = static_cast<int64_t>(slice) * KS;
  grid_dep_wait();    // Xq comes from the previous kernel
  grid_dep_launch();  // the finalize kernel may start launching

  // stage Xq[:, k0 : k0+KS] (tokens >= T and columns >= K are zero)
  const int64_t vec_per_row = KS / 16;
  for (int64_t i = threadIdx.x; i < NT * 8 * vec_per_row; i += THREADS) {
    const int tok = static_cast<int>(i / vec_per_row);
    const int64_t c16 = i - tok * vec_per_row;
    const int64_t k = k0 + c16 * 16;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (tok < T && k < K) v = ldg_v4(Xq + static_cast<int64_t>(tok) * K + k);
    *reinterpret_cast<uint4*>(sm + tok * pitch + c16 * 16) = v;
  }
  __syncthreads();

  int32_t* red = reinterpret_cast<int32_t*>(sm + NT * 8 * pitch);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, q = lane & 3;
  const int64_t kw = KS / WARPS;
  const int steps = static_cast<int>(kw / 64);
  const int64_t n_tiles = (N + ROWS - 1) / ROWS;

  for (int64_t tile = cta_in_slice; tile < n_tiles; tile += ctas_in_slice) {
    const int64_t n0 = tile * ROWS;
    const int64_t ra = n0 + g, rb = n0 + g + 8;
    const int8_t* pa = CB + ra * K;
    const int8_t* pb = CB + rb * K;
    const bool va = ra < N, vb = rb < N;
    int c[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0;

    constexpr int U = 4;  // steps in flight
    for (int st0 = 0; st0 < steps; st0 += U) {
      uint4 A0[U], A1[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int64_t ks = static_cast<int64_t>(warp) * kw + (st0 + u) * 64 + q * 16;
        const int64_t k = k0 + ks;
        const bool in = (st0 + u < steps) && (k < K);
        A0[u] = (in && va) ? ldg_stream_v4(pa + k) : make_uint4(0u, 0u, 0u, 0u);
        A1[u] = (in && vb) ? ldg_stream_v4(pb + k) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < U; ++u) {
        if (st0 + u < steps) {
          const int64_t ks = static_cast<int64_t>(warp) * kw + (st0 + u) * 64 + q * 16;
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            const uint4 B = *reinterpret_cast<const uint4*>(sm + (nt * 8 + g) * pitch + ks);
            mma_s8_16816(c[nt], A0[u].x, A1[u].x, A0[u].y, A1[u].y, B.x, B.y);
            mma_s8_16816(c[nt], A0[u].z, A1[u].z, A0[u].w, A1[u].w, B.z, B.w);
          }
        }
      }
    }
    // c[nt][0..3] = (row g, tok nt*8+2q), (row g, tok +1), (row g+8, tok), (row g+8, tok+1)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      int32_t* rw = red + (warp * ROWS) * (NT * 8);
      rw[g * (NT * 8) + nt * 8 + 2 * q] = c[nt][0];
      rw[g * (NT * 8) + nt * 8 + 2 * q + 1] = c[nt][1];
      rw[(g + 8) * (NT * 8) + nt * 8 + 2 * q] = c[nt][2];
      rw[(g + 8) * (NT * 8) + nt * 8 + 2 * q + 1] = c[nt][3];
    }
    __syncthreads();
    for (int i = threadIdx.x; i < ROWS * NT * 8; i += THREADS) {
      const int rr = i / (NT * 8), tok = i - rr * (NT * 8);
      int32_t sum = 0;
#pragma unroll
      for (int w = 0; w < WARPS; ++w) sum += red[(w * ROWS + rr) * (NT * 8) + tok];
      const int64_t n = n0 + rr;
      if (tok < T && n < N) P[(static_cast<int64_t>(slice) * T + tok) * N + n] = sum;
    }
    __syncthreads();
  }
}

// One thread per output (t, n) -- grid.y is the token: sum the K-slice partials (exact
// int32), then dequantise, add the outlier part (CB read straight through the index list,
// 8 loads in flight) and the bias.  kRaw writes the int32 sum.
template <bool kRaw>
__global__ void __launch_bounds__(256)
    gemv_finalize_kernel(const int32_t* __restrict__ P, int S, int T, int64_t N, int64_t K,
                         const float* __restrict__ SCx, const float* __restrict__ SCB,
                         const __half* __restrict__ bias, const int8_t* __restrict__ CB,
                         const int32_t* __restrict__ idx, const int32_t* __restrict__ n_o_ptr,
                         const __half* __restrict__ X_o, __half* __restrict__ C,
                         int32_t* __restrict__ acc_out) {
  const int64_t n = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int t = blockIdx.y;
  grid_dep_wait();    // the partial sums come from the previous kernel
  if (n >= N) return;
  int32_t acc = 0;
  for (int s = 0; s < S; ++s) acc += __ldcs(P + (static_cast<int64_t>(s) * T + t) * N + n);
  if (kRaw) {
    acc_out[static_cast<int64_t>(t) * N + n] = acc;
    return;
  }
  const int n_o = (n_o_ptr == nullptr) ? 0 : *n_o_ptr;
  float o = 0.0f;
  for (int j0 = 0; j0 < n_o; j0 += 8) {
    float cb[8], xo[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u;
      cb[u] = 0.0f;
      xo[u] = 0.0f;
      if (j < n_o) {
        cb[u] = static_cast<float>(CB[n * K + __ldg(idx + j)]);
        xo[u] = __half2float(X_o[(static_cast<int64_t>(j >> 6) * T + t) * 64 + (j & 63)]);
      }
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) o = fmaf(xo[u], cb[u], o);
  }
  const float ws = __ldg(SCB + n) * (1.0f / 127.0f);
  const float bn = bias ? __half2float(bias[n]) : 0.0f;
  const float part = fmaf(static_cast<float>(acc), __ldg(SCx + t) * (1.0f / 127.0f), o);
  C[static_cast<int64_t>(t) * N + n] = __float2half_rn(fmaf(part, ws, bn));
}

}  // namespace gemv
}  // namespace i8

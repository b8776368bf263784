// quant.cuh -- the HBM-bound passes over X and W:
//   outlier_scan_kernel    step 1: column OR of |x| >= threshold into a packed mask
//   compact_kernel         step 1: mask -> ascending outlier index list + count
//   quantize_rows_kernel   steps 2/3: row absmax (over the non-outlier columns) and int8
//                          codes; for the hidden states also the fp16 outlier slice X_o
//   gather_outlier_weights_kernel  step 6 operand: CB[:, idx] as exact fp16, chunk-major
// Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at
// scale" (Hugging Face blog), sections "absmax 量化", "LLM.int8() 的总结", "内部的 MatMul".
#pragma once

#include "common.cuh"

namespace i8 {

// ------------------------------------------------------------------ loads
__device__ __forceinline__ uint4 ldg_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ float2 h2f2(uint32_t u) {
  __half2 h = *reinterpret_cast<__half2*>(&u);
  return __half22float2(h);
}

// 8 fp16 values (one 16-byte vector, element i at the i-th lowest address) -> 8 bits of
// |x| >= thr.
__device__ __forceinline__ uint32_t outlier_bits8(const uint4 v, float thr) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t b = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = h2f2(w[i]);
    b |= (fabsf(f.x) >= thr ? 1u : 0u) << (2 * i);
    b |= (fabsf(f.y) >= thr ? 1u : 0u) << (2 * i + 1);
  }
  return b;
}

// ------------------------------------------------------------------ step 1: scan
constexpr int kScanThreads = 256;

// grid.x covers K in groups of 8 columns (one uint4 per thread), grid.y splits the rows.
__global__ void __launch_bounds__(kScanThreads)
    outlier_scan_kernel(const __half* __restrict__ X, int64_t T, int64_t K, float thr,
                        int64_t rows_per_cta, uint32_t* __restrict__ mask) {
  const int64_t groups = K >> 3;
  const int64_t g = static_cast<int64_t>(blockIdx.x) * kScanThreads + threadIdx.x;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_cta;
  const int64_t r1 = min(T, r0 + rows_per_cta);
  uint32_t bits = 0;
  if (g < groups) {
    const uint4* base = reinterpret_cast<const uint4*>(X) + g;
    int64_t r = r0;
    for (; r + 4 <= r1; r += 4) {
      uint4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) v[u] = ldg_v4(base + (r + u) * groups);
#pragma unroll
      for (int u = 0; u < 4; ++u) bits |= outlier_bits8(v[u], thr);
    }
    for (; r < r1; ++r) bits |= outlier_bits8(ldg_v4(base + r * groups), thr);
  }
  // four consecutive threads hold the 32 bits of one mask word
  uint32_t word = bits << (8 * (threadIdx.x & 3));
  word |= __shfl_xor_sync(0xffffffffu, word, 1);
  word |= __shfl_xor_sync(0xffffffffu, word, 2);
  if ((threadIdx.x & 3) == 0 && g < groups && word != 0u) atomicOr(mask + (g >> 2), word);
}

// One CTA: ascending list of set bits of the mask, and their count.
constexpr int kCompactThreads = 1024;

__global__ void __launch_bounds__(kCompactThreads)
    compact_kernel(const uint32_t* __restrict__ mask, int64_t words,
                   int32_t* __restrict__ idx, int32_t* __restrict__ n_o) {
  __shared__ int32_t warp_tot[kCompactThreads / 32];
  __shared__ int32_t carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int64_t base = 0; base < words; base += kCompactThreads) {
    const int64_t w = base + threadIdx.x;
    uint32_t word = (w < words) ? mask[w] : 0u;
    const int cnt = __popc(word);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int v = warp_tot[lane];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
      }
      warp_tot[lane] = v;  // inclusive prefix over warps
    }
    __syncthreads();
    int pos = carry + (warp > 0 ? warp_tot[warp - 1] : 0) + incl - cnt;
    while (word) {
      const int b = __ffs(word) - 1;
      idx[pos++] = static_cast<int32_t>(w * 32 + b);
      word &= word - 1u;
    }
    __syncthreads();
    if (threadIdx.x == 0) carry += warp_tot[kCompactThreads / 32 - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_o = carry;
}

// ------------------------------------------------------------------ steps 2 and 3
constexpr int kQuantThreads = 256;
constexpr int kQuantCacheVec = 8;  // 16-byte vectors per thread kept in registers

__device__ __forceinline__ float absmax8(const uint4 v, uint32_t skip) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.0f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = h2f2(w[i]);
    if (!((skip >> (2 * i)) & 1u)) m = fmaxf(m, fabsf(f.x));
    if (!((skip >> (2 * i + 1)) & 1u)) m = fmaxf(m, fabsf(f.y));
  }
  return m;
}

__device__ __forceinline__ uint2 codes8(const uint4 v, uint32_t skip, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    float2 f = h2f2(w[i]);
    int c0 = ((skip >> (2 * i)) & 1u) ? 0 : quant_code(f.x, s);
    int c1 = ((skip >> (2 * i + 1)) & 1u) ? 0 : quant_code(f.y, s);
    uint32_t pair = (static_cast<uint32_t>(c0) & 0xffu) | ((static_cast<uint32_t>(c1) & 0xffu) << 8);
    out[i >> 1] |= pair << (16 * (i & 1));
  }
  return make_uint2(out[0], out[1]);
}

__device__ __forceinline__ uint32_t skip_bits8(const uint32_t* mask, int64_t v) {
  return mask ? ((__ldg(mask + (v >> 2)) >> (8 * (v & 3))) & 0xffu) : 0u;
}

// One CTA per row of A [R, K].  mask (nullable) marks excluded columns (coded 0);
// idx/n_o/A_o (nullable) additionally gather the fp16 outlier slice of each row.
__global__ void __launch_bounds__(kQuantThreads)
    quantize_rows_kernel(const __half* __restrict__ A, int64_t R, int64_t K,
                         const uint32_t* __restrict__ mask, int8_t* __restrict__ Q,
                         float* __restrict__ scale, const int32_t* __restrict__ idx,
                         const int32_t* __restrict__ n_o_ptr, __half* __restrict__ A_o) {
  __shared__ float red[kQuantThreads / 32];
  const int64_t r = blockIdx.x;
  const int64_t nv = K >> 3;
  const uint4* row = reinterpret_cast<const uint4*>(A + r * K);
  uint4 cache[kQuantCacheVec];
  uint32_t skip[kQuantCacheVec];
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < kQuantCacheVec; ++i) {
    const int64_t v = threadIdx.x + static_cast<int64_t>(i) * kQuantThreads;
    cache[i] = make_uint4(0u, 0u, 0u, 0u);
    skip[i] = 0xffu;
    if (v < nv) {
      cache[i] = ldg_v4(row + v);
      skip[i] = skip_bits8(mask, v);
      amax = fmaxf(amax, absmax8(cache[i], skip[i]));
    }
  }
  for (int64_t v = threadIdx.x + static_cast<int64_t>(kQuantCacheVec) * kQuantThreads; v < nv;
       v += kQuantThreads)
    amax = fmaxf(amax, absmax8(ldg_v4(row + v), skip_bits8(mask, v)));

  amax = warp_max(amax);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = red[0];
#pragma unroll
  for (int w = 1; w < kQuantThreads / 32; ++w) amax = fmaxf(amax, red[w]);

  const float s = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
  uint2* qrow = reinterpret_cast<uint2*>(Q + r * K);
#pragma unroll
  for (int i = 0; i < kQuantCacheVec; ++i) {
    const int64_t v = threadIdx.x + static_cast<int64_t>(i) * kQuantThreads;
    if (v < nv) qrow[v] = codes8(cache[i], skip[i], s);
  }
  for (int64_t v = threadIdx.x + static_cast<int64_t>(kQuantCacheVec) * kQuantThreads; v < nv;
       v += kQuantThreads)
    qrow[v] = codes8(ldg_v4(row + v), skip_bits8(mask, v), s);
  if (threadIdx.x == 0) scale[r] = amax;

  if (A_o != nullptr) {
    const int n_o = *n_o_ptr;
    const int padded = (n_o + 63) & ~63;
    for (int j = threadIdx.x; j < padded; j += kQuantThreads) {
      __half v = __float2half_rn(0.0f);
      if (j < n_o) v = A[r * K + idx[j]];
      A_o[(static_cast<int64_t>(j >> 6) * R + r) * 64 + (j & 63)] = v;
    }
  }
}

// ------------------------------------------------------------------ step 6 operand
// CB_o(n, j) = (fp16) CB[n, idx[j]] (exact: |CB| <= 127), chunk-major [ceil(n_o/64)][N][64],
// zero for j >= n_o.  One warp per (chunk, row); each lane writes two adjacent halves.
__global__ void __launch_bounds__(256)
    gather_outlier_weights_kernel(const int8_t* __restrict__ CB, int64_t N, int64_t K,
                                  const int32_t* __restrict__ idx,
                                  const int32_t* __restrict__ n_o_ptr,
                                  __half* __restrict__ CB_o) {
  const int n_o = *n_o_ptr;
  const int64_t chunks = (n_o + 63) >> 6;
  const int64_t items = chunks * N;
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t it = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
       it < items; it += nwarps) {
    const int64_t c = it / N, n = it - c * N;
    const int64_t j0 = c * 64 + 2 * lane;
    float v0 = 0.0f, v1 = 0.0f;
    if (j0 < n_o) v0 = static_cast<float>(CB[n * K + idx[j0]]);
    if (j0 + 1 < n_o) v1 = static_cast<float>(CB[n * K + idx[j0 + 1]]);
    reinterpret_cast<__half2*>(CB_o + (c * N + n) * 64)[lane] = __floats2half2_rn(v0, v1);
  }
}

}  // namespace i8

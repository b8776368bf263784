// quant.cuh -- the HBM-bound passes over X and W:
//   outlier_scan_kernel    step 1: column OR of |x| >= threshold into a packed mask
//   compact_kernel         step 1: mask -> ascending outlier index list + count
//   quantize_rows_kernel   steps 2/3: row absmax (over the non-outlier columns) and int8
//                          codes; for the hidden states also the fp16 outlier slice X_o
//   quantize_weight_kernel step 3 for a whole weight: rows streamed through shared memory
//   prepare_kernel         steps 1 and 2 fused (one read of X), plus the fp16 outlier
//                          slices of X and of CB for step 6 (CB's kept across calls in an
//                          outlier cache when the caller provides one)
// Both quantisers also produce the e4m3 codes of the FP8 variant (scale 448 / absmax,
// nearest-even e4m3 rounding) when asked.
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

// Largest |x| of 8 fp16 values, as a float (exact: the fp16 maximum of the absolute values).
__device__ __forceinline__ float group_absmax(const uint4 v) {
  const __half2 a = __habs2(*reinterpret_cast<const __half2*>(&v.x));
  const __half2 b = __habs2(*reinterpret_cast<const __half2*>(&v.y));
  const __half2 c = __habs2(*reinterpret_cast<const __half2*>(&v.z));
  const __half2 d = __habs2(*reinterpret_cast<const __half2*>(&v.w));
  const __half2 m = __hmax2(__hmax2(a, b), __hmax2(c, d));
  return fmaxf(__low2float(m), __high2float(m));
}

// outlier_bits8 through the group's maximum first: most groups hold no value at the
// threshold and cost a few packed fp16 instructions.
__device__ __forceinline__ uint32_t outlier_bits8_fast(const uint4 v, float thr) {
  return group_absmax(v) >= thr ? outlier_bits8(v, thr) : 0u;
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
      for (int u = 0; u < 4; ++u) bits |= outlier_bits8_fast(v[u], thr);
    }
    for (; r < r1; ++r) bits |= outlier_bits8_fast(ldg_v4(base + r * groups), thr);
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

// int8 codes of 8 fp16 values (element i at the i-th lowest address) at scale s; excluded
// columns (skip bit i) give code 0.  Byte permutes gather the codes' low bytes.
__device__ __forceinline__ uint2 codes8(const uint4 v, uint32_t skip, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t c[8];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = h2f2(w[i]);
    c[2 * i] = ((skip >> (2 * i)) & 1u) ? 0u : quant_code_byte(f.x, s);
    c[2 * i + 1] = ((skip >> (2 * i + 1)) & 1u) ? 0u : quant_code_byte(f.y, s);
  }
  const uint32_t lo = __byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040),
                                  0x5410);
  const uint32_t hi = __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040),
                                  0x5410);
  return make_uint2(lo, hi);
}

// e4m3 variant: the codes of 8 fp16 values are the e4m3 roundings (nearest, ties to even;
// magnitudes beyond 448 saturate) of fl32(x * s); excluded columns, and every column of
// a row whose scale is 0, give code 0.  Two values per conversion instruction: the
// second source goes to the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ uint2 codes8_e4m3(const uint4 v, uint32_t skip, float s) {
  if (s == 0.0f) return make_uint2(0u, 0u);
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2] = {0u, 0u};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = h2f2(w[i]);
    const float p0 = ((skip >> (2 * i)) & 1u) ? 0.0f : __fmul_rn(f.x, s);
    const float p1 = ((skip >> (2 * i + 1)) & 1u) ? 0.0f : __fmul_rn(f.y, s);
    out[i >> 1] |= e4m3x2(p0, p1) << (16 * (i & 1));
  }
  return make_uint2(out[0], out[1]);
}

// codes of 8 values in the layer's code format (int8, or e4m3 when e4m3 is set)
__device__ __forceinline__ uint2 codes8_fmt(const uint4 v, uint32_t skip, float s, bool e4m3) {
  return e4m3 ? codes8_e4m3(v, skip, s) : codes8(v, skip, s);
}

// largest code magnitude of the format: the absmax maps onto it
__device__ __forceinline__ float code_max(bool e4m3) { return e4m3 ? 448.0f : 127.0f; }

// fp16 value of one weight code (an int8 code, or an e4m3 code in the low byte of c)
__device__ __forceinline__ __half code_to_half(int c, bool e4m3) {
  if (!e4m3) return __int2half_rn(c);
  uint32_t h;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(c & 0xff)));
  return __ushort_as_half(static_cast<unsigned short>(h & 0xffffu));
}

// fp16 values of two weight codes (bytes b0, b1; only their low bytes count) as a half2
// (b0 in the low half).  int8: with u = c + 128 = (byte ^ 0x80), the fp16 pattern
// 0x6400 | u is 1024 + u exactly (a 10-bit mantissa at exponent 10), and subtracting
// 1152 leaves c exactly -- integer operations and one packed subtraction instead of two
// conversions.  e4m3: the packed hardware conversion.
__device__ __forceinline__ __half2 codes_to_half2(uint32_t b0, uint32_t b1, bool e4m3) {
  const uint32_t pair = __byte_perm(b0, b1, 0x0040);  // b0 in byte 0, b1 in byte 1
  if (e4m3) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(static_cast<uint16_t>(pair)));
    return *reinterpret_cast<__half2*>(&h);
  }
  uint32_t w = __byte_perm(pair, 0x64646464u, 0x5140) ^ 0x00800080u;
  const __half2 biased = *reinterpret_cast<__half2*>(&w);
  return __hsub2(biased, __halves2half2(__ushort_as_half(0x6480), __ushort_as_half(0x6480)));
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
                         const int32_t* __restrict__ n_o_ptr, __half* __restrict__ A_o,
                         bool e4m3 = false) {
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

  const float s = amax > 0.0f ? __fdiv_rn(code_max(e4m3), amax) : 0.0f;
  uint2* qrow = reinterpret_cast<uint2*>(Q + r * K);
#pragma unroll
  for (int i = 0; i < kQuantCacheVec; ++i) {
    const int64_t v = threadIdx.x + static_cast<int64_t>(i) * kQuantThreads;
    if (v < nv) qrow[v] = codes8_fmt(cache[i], skip[i], s, e4m3);
  }
  for (int64_t v = threadIdx.x + static_cast<int64_t>(kQuantCacheVec) * kQuantThreads; v < nv;
       v += kQuantThreads)
    qrow[v] = codes8_fmt(ldg_v4(row + v), skip_bits8(mask, v), s, e4m3);
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


// ====================================================================== fused pass
// prepare_kernel: steps 1 and 2 in one launch, reading X from HBM once when the rows of
// each CTA fit in its shared memory (re-reading, mostly from L2, the rows that do not):
//   phase 1  each CTA pulls its block of rows into shared memory with bulk (TMA) copies,
//            scans it, and ORs its column bits into the global mask;
//   barrier  one grid-wide barrier (every CTA is resident: one CTA per SM; the wait is
//            bounded like every other wait in this library);
//   phase 2  every CTA reads the final mask and builds the ascending outlier index list
//            in its own shared memory; CTA 0 also writes it (and n_o) to global memory;
//   phase 3  all threads of the CTA walk its rows together: absmax over the non-outlier
//            columns, int8 codes, the fp16 outlier slice X_o;
//   phase 4  (GEMM path) the fp16 outlier slice of the weight, CB_o, for all N rows.
// The caller clears mask[0 .. words] (the last word is the barrier counter) beforehand.
constexpr int kPrepThreads = 512;
constexpr int kPrepWarps = kPrepThreads / 32;
constexpr int kPrepChunk = 32768;   // bytes per bulk copy of the row cache
constexpr int kPrepMaxChunks = 8;
constexpr int kPrepMaxIdx = 8192;    // outlier indices kept in shared memory
constexpr int kSpecMinRows = 8;      // cached rows from which a CTA quantises early
// Outlier cache header, 32-bit words: [0] valid, [1] n_o, [2] N, [3] K, [4..5] the CB
// device pointer (low, high), [6..7] spare, then the ceil(K/32) mask words of the cached set.
constexpr int kOcacheHdrWords = 8;

struct PrepArgs {
  const __half* X;
  int64_t T, K;
  float thr;
  uint32_t* mask;         // [words + 2]: mask, the barrier counter, the cache-update counter
  int32_t* idx_out;       // [K]
  int32_t* n_o_out;       // [1]
  int8_t* Xq;
  float* SCx;
  __half* X_o;            // chunk-major slice [ceil(K/64)][T][64]
  const int8_t* CB;       // [N, K] (phase 4) or NULL
  int64_t N;
  __half* CB_o;           // chunk-major slice [ceil(K/64)][N][64] or NULL
  // Outlier cache (NULL: none).  CB_o of a call whose outlier set (and weight) matches the
  // cached one is the cache's slice as it stands; otherwise it is gathered, into the cache
  // when n_o <= ocache_cols (which then keys it by this call's set), else into CB_o above.
  uint32_t* ocache;       // header (kOcacheHdrWords words, then the mask words)
  __half* ocache_CB_o;    // chunk-major slice [ocache_cols / 64][N][64]
  int64_t ocache_cols;    // capacity in columns, a multiple of 64
  int32_t* cbo_sel;       // out (may be NULL): 1 when this call's CB_o is the cache's slice
  int64_t rows_per_cta;
  int64_t cache_rows;     // rows of its block each CTA keeps in shared memory
  int64_t cache_bytes_all; // size of the row-cache region (reused by phase 4)
  uint64_t wait_limit_ns;
};

__host__ __device__ inline int g32_of(int64_t K) { return static_cast<int>(K / 16); }

__device__ __forceinline__ uint32_t ld_acquire_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// fast absmax of 8 fp16 values when none of them is excluded (exact in fp16)
__device__ __forceinline__ float absmax8_all(const uint4 v) {
  __half2 a = __habs2(*reinterpret_cast<const __half2*>(&v.x));
  __half2 b = __habs2(*reinterpret_cast<const __half2*>(&v.y));
  __half2 c = __habs2(*reinterpret_cast<const __half2*>(&v.z));
  __half2 d = __habs2(*reinterpret_cast<const __half2*>(&v.w));
  const __half2 m = __hmax2(__hmax2(a, b), __hmax2(c, d));
  return fmaxf(__low2float(m), __high2float(m));
}

__device__ __forceinline__ uint32_t scan_bits(const uint32_t* smask, int64_t g) {
  return (smask[g >> 2] >> (8 * (g & 3))) & 0xffu;
}

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "r"(addr));
  return v;
}

// 16-byte group v of a row held in shared memory (kShared, `base` a shared address) or in
// global memory (`gbase`).
template <bool kShared>
__device__ __forceinline__ uint4 row_vec(uint32_t base, const uint4* gbase, int v) {
  if (kShared) return lds_v4(base + static_cast<uint32_t>(v) * 16u);
  return ldg_v4(gbase + v);
}

// Max |x| over the non-outlier columns of groups start, start+step, ... of one row.
template <bool kShared>
__device__ __forceinline__ float row_absmax(uint32_t base, const uint4* gbase, int gpr, int start,
                                            int step, const uint32_t* smask) {
  float m0 = 0.0f, m1 = 0.0f, m2 = 0.0f, m3 = 0.0f;
  int v = start;
  for (; v + 3 * step < gpr; v += 4 * step) {
    const uint4 x0 = row_vec<kShared>(base, gbase, v);
    const uint4 x1 = row_vec<kShared>(base, gbase, v + step);
    const uint4 x2 = row_vec<kShared>(base, gbase, v + 2 * step);
    const uint4 x3 = row_vec<kShared>(base, gbase, v + 3 * step);
    const uint32_t k0 = scan_bits(smask, v), k1 = scan_bits(smask, v + step);
    const uint32_t k2 = scan_bits(smask, v + 2 * step), k3 = scan_bits(smask, v + 3 * step);
    m0 = fmaxf(m0, k0 ? absmax8(x0, k0) : absmax8_all(x0));
    m1 = fmaxf(m1, k1 ? absmax8(x1, k1) : absmax8_all(x1));
    m2 = fmaxf(m2, k2 ? absmax8(x2, k2) : absmax8_all(x2));
    m3 = fmaxf(m3, k3 ? absmax8(x3, k3) : absmax8_all(x3));
  }
  for (; v < gpr; v += step) {
    const uint32_t k = scan_bits(smask, v);
    const uint4 x = row_vec<kShared>(base, gbase, v);
    m0 = fmaxf(m0, k ? absmax8(x, k) : absmax8_all(x));
  }
  return fmaxf(fmaxf(m0, m1), fmaxf(m2, m3));
}

// The outlier values of one 16-byte group v of a row (its mask bits k != 0) into the
// row's fp16 outlier slice: the column of bit b has rank spre[v/4] + (mask bits below it),
// and rank j goes to xo[(j / 64) * cstride + j % 64].
__device__ __forceinline__ void group_outliers(const uint4 x, int v, uint32_t k,
                                               const uint32_t* smask, const int32_t* spre,
                                               __half* xo, int64_t cstride) {
  const uint32_t w = smask[v >> 2];
  const int sh = (v & 3) * 8;
  int j = spre[v >> 2] + __popc(w & ((1u << sh) - 1u));
  while (k) {
    const int b = __ffs(k) - 1;
    k &= k - 1u;
    const uint32_t pr = (b & 4) ? ((b & 2) ? x.w : x.z) : ((b & 2) ? x.y : x.x);
    const uint32_t hw = pr >> (16 * (b & 1));
    xo[static_cast<int64_t>(j >> 6) * cstride + (j & 63)] =
        __ushort_as_half(static_cast<unsigned short>(hw & 0xffffu));
    ++j;
  }
}

// codes (int8, or e4m3) of groups start, start+step, ... of one row; with xo non-NULL, the
// row's outlier values also go into its fp16 outlier slice (group_outliers).
template <bool kShared>
__device__ __forceinline__ void row_codes(uint32_t base, const uint4* gbase, uint2* q, int gpr,
                                          int start, int step, const uint32_t* smask, float s,
                                          bool e4m3, const int32_t* spre = nullptr,
                                          __half* xo = nullptr, int64_t cstride = 0) {
  int v = start;
  for (; v + 3 * step < gpr; v += 4 * step) {
    const uint4 x0 = row_vec<kShared>(base, gbase, v);
    const uint4 x1 = row_vec<kShared>(base, gbase, v + step);
    const uint4 x2 = row_vec<kShared>(base, gbase, v + 2 * step);
    const uint4 x3 = row_vec<kShared>(base, gbase, v + 3 * step);
    const uint32_t k0 = scan_bits(smask, v), k1 = scan_bits(smask, v + step);
    const uint32_t k2 = scan_bits(smask, v + 2 * step), k3 = scan_bits(smask, v + 3 * step);
    q[v] = codes8_fmt(x0, k0, s, e4m3);
    q[v + step] = codes8_fmt(x1, k1, s, e4m3);
    q[v + 2 * step] = codes8_fmt(x2, k2, s, e4m3);
    q[v + 3 * step] = codes8_fmt(x3, k3, s, e4m3);
    if (xo != nullptr && (k0 | k1 | k2 | k3) != 0u) {
      if (k0) group_outliers(x0, v, k0, smask, spre, xo, cstride);
      if (k1) group_outliers(x1, v + step, k1, smask, spre, xo, cstride);
      if (k2) group_outliers(x2, v + 2 * step, k2, smask, spre, xo, cstride);
      if (k3) group_outliers(x3, v + 3 * step, k3, smask, spre, xo, cstride);
    }
  }
  for (; v < gpr; v += step) {
    const uint4 x = row_vec<kShared>(base, gbase, v);
    const uint32_t k = scan_bits(smask, v);
    q[v] = codes8_fmt(x, k, s, e4m3);
    if (xo != nullptr && k != 0u) group_outliers(x, v, k, smask, spre, xo, cstride);
  }
}

// Column of the j-th outlier (j < n_o) from the mask words and their exclusive popcount
// prefix (spre[words] = n_o): the last word whose prefix is <= j holds it.
__device__ __forceinline__ int32_t nth_outlier(const uint32_t* smask, const int32_t* spre,
                                               int64_t words, int j) {
  int64_t lo = 0, hi = words - 1;
  while (lo < hi) {
    const int64_t mid = (lo + hi + 1) >> 1;
    if (spre[mid] <= j)
      lo = mid;
    else
      hi = mid - 1;
  }
  uint32_t m = smask[lo];
  for (int k = j - spre[lo]; k > 0; --k) m &= m - 1u;
  return static_cast<int32_t>(lo * 32 + (__ffs(m) - 1));
}

// kE4M3: e4m3 codes (scale 448 / absmax) instead of int8 (the layer's code format, fixed at
// compile time so that each variant carries only its own code path).
template <bool kE4M3>
__global__ void __launch_bounds__(kPrepThreads, 1) prepare_kernel(const PrepArgs p) {
  extern __shared__ __align__(128) uint8_t psm[];
  const int64_t K = p.K;
  const int64_t words = (K + 31) / 32;
  const int64_t gpr = K / 8;  // 16-byte groups per row
  // shared memory: [row cache][mask words][prefix words + 1][first kPrepMaxIdx indices]
  // [speculative row scales][speculative block maxima, 128 columns per block, cached rows];
  // indices past kPrepMaxIdx are found from the mask and its prefix
  const size_t cache_bytes = static_cast<size_t>(p.cache_rows) * static_cast<size_t>(K) * 2;
  uint4* cache = reinterpret_cast<uint4*>(psm);
  uint32_t* smask = reinterpret_cast<uint32_t*>(psm + cache_bytes);
  int32_t* spre = reinterpret_cast<int32_t*>(smask + words);
  int32_t* sidx = spre + words + 2;  // 8-byte aligned: pairs of indices load as one word
  float* samax = reinterpret_cast<float*>(sidx + kPrepMaxIdx);   // [rows_per_cta]
  float* sbm = samax + p.rows_per_cta;                           // [cache_rows][nblk]
  __shared__ __align__(8) uint64_t s_bar[kPrepMaxChunks];
  __shared__ __align__(8) uint64_t s_rbar[kPrepWarps];  // phase 4 row buffers
  __shared__ __align__(8) uint64_t s_sbar[kPrepWarps];  // phase 3 row slots
  __shared__ int s_fail;
  __shared__ int s_gfail;  // phase 4 gave up on a wait: the cache is left invalid
  __shared__ int s_last;
  __shared__ int s_wsum[kPrepWarps];
  __shared__ float s_red[kPrepWarps];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * p.rows_per_cta;
  const int64_t r1 = min(p.T, r0 + p.rows_per_cta);
  const int64_t nrows = r1 > r0 ? r1 - r0 : 0;
  const int64_t ncached = min(nrows, p.cache_rows);
  const int64_t cbytes = ncached * K * 2;
  const int nchunks = static_cast<int>((cbytes + kPrepChunk - 1) / kPrepChunk);

  // ------------------------------------------------ phase 1: scan (and cache) the rows
  if (tid == 0) {
    s_fail = 0;
    s_gfail = 0;
    for (int c = 0; c < nchunks; ++c) mbar_init(smem_u32(&s_bar[c]), 1);
    for (int c = 0; c < kPrepWarps; ++c) mbar_init(smem_u32(&s_rbar[c]), 1);
    for (int c = 0; c < kPrepWarps; ++c) mbar_init(smem_u32(&s_sbar[c]), 1);
    fence_mbar_init();
  }
  for (int64_t w = tid; w < words; w += kPrepThreads) smask[w] = 0u;
  __syncthreads();
  if (tid == 0) {
    const uint8_t* src = reinterpret_cast<const uint8_t*>(p.X + r0 * K);
    for (int c = 0; c < nchunks; ++c) {
      const int64_t off = static_cast<int64_t>(c) * kPrepChunk;
      const uint32_t bytes = static_cast<uint32_t>(min(static_cast<int64_t>(kPrepChunk), cbytes - off));
      mbar_arrive_expect_tx(smem_u32(&s_bar[c]), bytes);
      bulk_load(smem_u32(psm + off), src + off, bytes, smem_u32(&s_bar[c]));
    }
  }
  // rows beyond the cache: scanned straight from global memory while the copies land
  {
    const uint4* src = reinterpret_cast<const uint4*>(p.X + (r0 + ncached) * K);
    const int64_t nvec = (nrows - ncached) * gpr;
    int64_t v = tid;
    for (; v + 3 * kPrepThreads < nvec; v += 4 * kPrepThreads) {
      uint4 x[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) x[u] = ldg_v4(src + v + u * kPrepThreads);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const uint32_t f = outlier_bits8_fast(x[u], p.thr);
        if (f) {
          const int64_t g = (v + u * kPrepThreads) % gpr;
          atomicOr(smask + (g >> 2), f << (8 * (g & 3)));
        }
      }
    }
    for (; v < nvec; v += kPrepThreads) {
      const uint32_t f = outlier_bits8_fast(ldg_v4(src + v), p.thr);
      if (f) {
        const int64_t g = v % gpr;
        atomicOr(smask + (g >> 2), f << (8 * (g & 3)));
      }
    }
  }
  // Cached rows.  A CTA that keeps at least kSpecMinRows rows in shared memory quantises
  // them speculatively before the grid barrier: one warp per row, as soon as the chunks
  // holding it have landed, scans the row (its outlier bits go into the CTA's mask), takes
  // the largest |x| below the threshold per 128-column block and over the row, and writes
  // the row's codes at that scale.  The final mask can only add columns in which this
  // row's elements are below the threshold; phase 3 takes the true scale from the block
  // maxima (re-reading only the blocks that hold outlier columns) and, when it is the
  // speculative one, only clears the codes of the outlier columns.  Other CTAs scan each
  // chunk as it lands and quantise in phase 3.
  const bool spec = ncached >= kSpecMinRows;
  const int nblk = static_cast<int>((gpr + 15) / 16);
  if (spec) {
    int no_abort = 0;
    const int g32 = static_cast<int>(gpr);
    const uint32_t cache_s = smem_u32(cache);
    for (int64_t i = warp; i < ncached; i += kPrepWarps) {
      const int c_first = static_cast<int>(i * K * 2 / kPrepChunk);
      const int c_last = static_cast<int>(((i + 1) * K * 2 - 1) / kPrepChunk);
      bool got = true;
      for (int c = c_first; c <= c_last; ++c)
        got = mbar_wait(smem_u32(&s_bar[c]), 0u, &no_abort, p.wait_limit_ns) && got;
      if (!__all_sync(0xffffffffu, got)) {
        if (lane == 0) s_fail = 1;
        continue;
      }
      const uint32_t rbase = cache_s + static_cast<uint32_t>(i * gpr * 16);
      float mrow = 0.0f;
      for (int g0 = 0; g0 < g32; g0 += 32) {  // 32 groups: two blocks, one per half-warp
        const int g = g0 + lane;
        float m = 0.0f;
        if (g < g32) {
          const uint4 x = lds_v4(rbase + static_cast<uint32_t>(g) * 16u);
          m = group_absmax(x);
          if (m >= p.thr) {   // rare: a value at the threshold in this group
            const uint32_t f = outlier_bits8(x, p.thr);
            atomicOr(smask + (g >> 2), f << (8 * (g & 3)));
            m = absmax8(x, f);
          }
        }
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 8));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        if ((lane & 15) == 0 && g < g32) sbm[i * nblk + (g >> 4)] = m;
        mrow = fmaxf(mrow, m);
      }
      mrow = fmaxf(mrow, __shfl_xor_sync(0xffffffffu, mrow, 16));
      __syncwarp();  // every lane sees the row's own outlier bits in the mask
      // codes at the speculative scale; columns already in the CTA's mask (the row's own
      // outliers among them) get code 0, as every column of the final mask must
      const float sc = mrow > 0.0f ? __fdiv_rn(code_max(kE4M3), mrow) : 0.0f;
      row_codes<true>(rbase, nullptr, reinterpret_cast<uint2*>(p.Xq + (r0 + i) * K), g32, lane,
                      32, smask, sc, kE4M3);
      if (lane == 0) samax[i] = mrow;
    }
  } else {
    int no_abort = 0;
    for (int c = 0; c < nchunks; ++c) {
      const bool got = mbar_wait(smem_u32(&s_bar[c]), 0u, &no_abort, p.wait_limit_ns);
      if (!got) s_fail = 1;
      const int64_t v0 = static_cast<int64_t>(c) * (kPrepChunk / 16);
      const int64_t v1 = min(v0 + static_cast<int64_t>(kPrepChunk / 16), cbytes / 16);
      for (int64_t v = v0 + tid; v < v1; v += kPrepThreads) {
        const uint32_t f = got ? outlier_bits8_fast(cache[v], p.thr) : 0u;
        if (f) {
          const int64_t g = v % gpr;
          atomicOr(smask + (g >> 2), f << (8 * (g & 3)));
        }
      }
    }
  }
  __syncthreads();
  for (int64_t w = tid; w < words; w += kPrepThreads)
    if (smask[w]) atomicOr(p.mask + w, smask[w]);
  grid_dep_launch();  // the GEMM / GEMV may start launching (it waits for our writes)

  // ------------------------------------------------ grid barrier (bounded)
  __syncthreads();
  if (tid == 0) {
    uint32_t* counter = p.mask + words;
    __threadfence();
    atomicAdd(counter, 1u);
    const uint32_t target = gridDim.x;
    if (ld_acquire_gpu(counter) < target) {
      const uint64_t t0 = globaltimer_ns();
      for (uint32_t it = 1;; ++it) {
        if (ld_acquire_gpu(counter) >= target) break;
        if ((it & 63u) == 0u && globaltimer_ns() - t0 > p.wait_limit_ns) {
          raise_error(kErrWaitTimeout);
          s_fail = 1;
          break;
        }
      }
    }
    __threadfence();
  }
  __syncthreads();
  if (s_fail) {
    if (tid == 0) {
      raise_error(kErrWaitTimeout);
      int no_abort = 0;  // let the copies in flight land before the CTA exits (bounded)
      for (int c = 0; c < nchunks; ++c)
        mbar_wait(smem_u32(&s_bar[c]), 0u, &no_abort, p.wait_limit_ns);
    }
    __syncthreads();
    return;
  }

  // ------------------------------------------------ phase 2: final mask, index list
  // exclusive prefix of the per-word popcounts, blocks of kPrepThreads words at a time
  int carry = 0;
  for (int64_t base = 0; base < words; base += kPrepThreads) {
    const int64_t w = base + tid;
    uint32_t m = 0u;
    if (w < words) {
      m = __ldcg(p.mask + w);
      smask[w] = m;
    }
    const int c = __popc(m);
    int incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) s_wsum[warp] = incl;
    __syncthreads();
    int before = 0, total = 0;
#pragma unroll
    for (int w2 = 0; w2 < kPrepWarps; ++w2) {
      const int x = s_wsum[w2];
      before += (w2 < warp) ? x : 0;
      total += x;
    }
    if (w < words) spre[w] = carry + before + incl - c;
    carry += total;
    __syncthreads();
  }
  if (tid == 0) spre[words] = carry;
  const int n_o = carry;
  for (int64_t w = tid; w < words; w += kPrepThreads) {
    uint32_t m = smask[w];
    int pos = spre[w];
    while (m) {
      const int b = __ffs(m) - 1;
      const int32_t col = static_cast<int32_t>(w * 32 + b);
      if (pos < kPrepMaxIdx) sidx[pos] = col;
      if (blockIdx.x == 0) p.idx_out[pos] = col;
      ++pos;
      m &= m - 1u;
    }
  }
  __syncthreads();
  if (blockIdx.x == 0 && tid == 0) *p.n_o_out = n_o;
  auto idx_at = [&](int j) -> int64_t {
    return j < kPrepMaxIdx ? sidx[j] : nth_outlier(smask, spre, words, j);
  };

  // Outlier cache: cmode 0 = not used, 1 = hit (CB_o is the cache's slice as it stands),
  // 2 = miss (gather into the cache's slice, then key the cache by this call's set).  Every
  // CTA reads the same header and the same final mask, so all take the same decision; a
  // missing CTA clears the valid word before it writes the slice, which can only turn the
  // decision of a CTA that reads the header later into the miss it takes anyway.
  int cmode = 0;
  if (p.ocache != nullptr && p.CB != nullptr && n_o > 0 && n_o <= p.ocache_cols) {
    const uint32_t* h = p.ocache;
    bool same = true;
    if (tid == 0) {
      const uint64_t cbp = reinterpret_cast<uint64_t>(p.CB);
      same = __ldcg(h + 0) == 1u && __ldcg(h + 1) == static_cast<uint32_t>(n_o) &&
             __ldcg(h + 2) == static_cast<uint32_t>(p.N) &&
             __ldcg(h + 3) == static_cast<uint32_t>(K) &&
             __ldcg(h + 4) == static_cast<uint32_t>(cbp) &&
             __ldcg(h + 5) == static_cast<uint32_t>(cbp >> 32);
    }
    for (int64_t w = tid; w < words; w += kPrepThreads)
      if (__ldcg(h + kOcacheHdrWords + w) != smask[w]) same = false;
    cmode = __syncthreads_and(same) ? 1 : 2;
    if (cmode == 2 && tid == 0) {
      __stcg(p.ocache, 0u);
      __threadfence();
    }
  }
  __half* const cbo = cmode != 0 ? p.ocache_CB_o : p.CB_o;
  const bool gather = cbo != nullptr && cmode != 1 && n_o > 0;
  if (blockIdx.x == 0 && tid == 0 && p.cbo_sel != nullptr) *p.cbo_sel = cmode != 0 ? 1 : 0;

  // The CB_o gather of phase 4 for few outlier columns (one warp per (chunk, row) item,
  // U4 items per batch) is bound by the latency of scattered byte reads of CB in HBM, so
  // each warp issues its first batch here and stores it after the quantisation: those
  // loads are in flight while the rows are quantised.
  constexpr int U4 = 8;
  const int64_t chunks4 = (n_o + 63) >> 6;
  const int64_t nbuf4 = min(static_cast<int64_t>(kPrepWarps), p.cache_bytes_all / K);
  const bool few4 = gather && !(static_cast<int64_t>(n_o) * 64 >= K && nbuf4 > 0);
  const int64_t items4 = chunks4 * p.N;
  const int64_t nw4 = static_cast<int64_t>(gridDim.x) * kPrepWarps;
  const int64_t first4 = (static_cast<int64_t>(blockIdx.x) * kPrepWarps + warp) * U4;
  // (the loaded bytes stay unconverted until the store, so nothing waits on them before)
  auto gather_load = [&](int64_t it0, int (&v0)[U4], int (&v1)[U4]) {
#pragma unroll
    for (int u = 0; u < U4; ++u) {
      const int64_t it = it0 + u;
      v0[u] = 0;
      v1[u] = 0;
      if (it < items4) {
        const int64_t c = it / p.N, n = it - c * p.N;
        const int64_t j0 = c * 64 + 2 * lane;
        if (j0 < n_o) v0[u] = reinterpret_cast<const uint8_t*>(p.CB)[n * K + idx_at(j0)];
        if (j0 + 1 < n_o) v1[u] = reinterpret_cast<const uint8_t*>(p.CB)[n * K + idx_at(j0 + 1)];
      }
    }
  };
  auto gather_store = [&](int64_t it0, const int (&v0)[U4], const int (&v1)[U4]) {
#pragma unroll
    for (int u = 0; u < U4; ++u) {
      const int64_t it = it0 + u;
      if (it < items4) {
        const int64_t c = it / p.N, n = it - c * p.N;
        reinterpret_cast<__half2*>(cbo + (c * p.N + n) * 64)[lane] =
            codes_to_half2(static_cast<uint32_t>(v0[u]), static_cast<uint32_t>(v1[u]), kE4M3);
      }
    }
  };
  int pv0[U4], pv1[U4];
  if (few4) gather_load(first4, pv0, pv1);

  // ------------------------------------------------ phase 3: quantise
  // Rows go in rounds of (16 / wpr) rows with wpr warps per row (wpr = 1 for 16 rows or
  // more; up to 16 for one row, as in decode batches).  Every warp walks the same rounds,
  // so the block barriers of the cross-warp reduction are uniform.  First the cached rows,
  // from shared memory; then the others.  Those come into the freed row cache by bulk copy,
  // one row per slot and round (each row is then read from shared memory for both its
  // maximum and its codes, instead of twice from global memory with a few loads in flight
  // per lane); without room for one row they are read from global memory.
  const int padded = (n_o + 63) & ~63;
  const int g32 = static_cast<int>(gpr);
  const uint32_t cache_s = smem_u32(cache);
  const int64_t row_bytes = gpr * 16;
  int nsl = 0;  // row slots for the uncached rows: a power of two, at most kPrepWarps
  {
    const int64_t cap = row_bytes > 0 ? p.cache_bytes_all / row_bytes : 0;
    while (nsl < kPrepWarps && 2 * (nsl > 0 ? nsl : 1) <= cap) nsl = nsl > 0 ? 2 * nsl : 2;
    if (nsl == 0 && cap >= 1) nsl = 1;
  }
  auto quantise_rows = [&](int64_t lo, int64_t hi, bool staged) {
    const int64_t n = hi - lo;
    int wpr = 1;
    while (wpr < kPrepWarps && wpr * 2 * n <= kPrepWarps) wpr *= 2;
    if (staged)
      while (kPrepWarps / wpr > nsl) wpr *= 2;
    const int rows_per_round = kPrepWarps / wpr;
    const int sub = warp % wpr;
    const int rr = warp / wpr;
    const int start = sub * 32 + lane, step = 32 * wpr;
    const int64_t rounds = (n + rows_per_round - 1) / rows_per_round;
    for (int64_t round = 0; round < rounds; ++round) {
      const int64_t i = lo + round * rows_per_round + rr;
      const bool have = i < hi;
      const bool cached = have && i < ncached;
      const int64_t t = r0 + i;
      uint32_t sbase = cache_s + static_cast<uint32_t>(i * row_bytes);
      const uint4* gbase = reinterpret_cast<const uint4*>(p.X + t * K);
      if (staged) {
        // the previous round's reads of the slots are done before they are written again
        __syncthreads();
        if (warp == 0 && lane < rows_per_round) {
          const int64_t il = lo + round * rows_per_round + lane;
          if (il < hi) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            const uint32_t bar = smem_u32(&s_sbar[lane]);
            mbar_arrive_expect_tx(bar, static_cast<uint32_t>(row_bytes));
            bulk_load(cache_s + static_cast<uint32_t>(lane * row_bytes), p.X + (r0 + il) * K,
                      static_cast<uint32_t>(row_bytes), bar);
          }
        }
        sbase = cache_s + static_cast<uint32_t>(rr * row_bytes);
        if (have) {
          int no_abort = 0;
          const bool got = mbar_wait(smem_u32(&s_sbar[rr]), static_cast<uint32_t>(round & 1),
                                     &no_abort, p.wait_limit_ns);
          if (!__all_sync(0xffffffffu, got) && lane == 0) s_gfail = 1;
        }
      }
      const bool in_smem = cached || (staged && have);
      const bool specrow = spec && cached;
      float amax = 0.0f;
      if (specrow) {
        // blocks free of outlier columns: their speculative maxima are exact; the others
        // are read again without the outlier columns
        for (int b = start; b < nblk; b += step) {
          const int ga = b * 16, gb = min(ga + 16, g32);
          bool dirty = false;
          for (int g = ga; g < gb; g += 4) dirty = dirty || smask[g >> 2] != 0u;
          if (!dirty) {
            amax = fmaxf(amax, sbm[i * nblk + b]);
          } else {
            for (int g = ga; g < gb; ++g) {
              const uint32_t k = scan_bits(smask, g);
              const uint4 x = lds_v4(sbase + static_cast<uint32_t>(g) * 16u);
              amax = fmaxf(amax, k ? absmax8(x, k) : absmax8_all(x));
            }
          }
        }
      } else if (in_smem) {
        amax = row_absmax<true>(sbase, gbase, g32, start, step, smask);
      } else if (have) {
        amax = row_absmax<false>(sbase, gbase, g32, start, step, smask);
      }
      amax = warp_max(amax);
      if (wpr > 1) {
        __syncthreads();
        if (lane == 0) s_red[warp] = amax;
        __syncthreads();
        for (int w2 = 0; w2 < wpr; ++w2) amax = fmaxf(amax, s_red[rr * wpr + w2]);
      }
      if (!have) continue;
      const float sc = amax > 0.0f ? __fdiv_rn(code_max(kE4M3), amax) : 0.0f;
      uint2* qrow = reinterpret_cast<uint2*>(p.Xq + t * K);
      __half* xo_row = p.X_o + t * 64;
      const int64_t cstride = p.T * 64;
      const bool stand = specrow && amax == samax[i] && static_cast<int64_t>(n_o) * 8 <= K;
      if (stand) {
        // the speculative codes stand: clear those of the outlier columns
        int8_t* qb = p.Xq + t * K;
        for (int j = start; j < n_o; j += step) qb[idx_at(j)] = 0;
      } else if (in_smem) {
        row_codes<true>(sbase, gbase, qrow, g32, start, step, smask, sc, kE4M3, spre, xo_row,
                        cstride);
      } else {
        row_codes<false>(sbase, gbase, qrow, g32, start, step, smask, sc, kE4M3, spre, xo_row,
                         cstride);
      }
      if (sub == 0 && lane == 0) p.SCx[t] = amax;
      // the row's outlier values into X_o (the codes pass above wrote them unless the
      // speculative codes stood; a cached row reads them from shared memory), and zeros up
      // to the next multiple of 64
      if (stand) {
        const __half* xrow = reinterpret_cast<const __half*>(cache + i * gpr);
        for (int j0 = start; j0 < n_o; j0 += 8 * step) {
          __half v[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = j0 + u * step;
            v[u] = __float2half_rn(0.0f);
            if (j < n_o) v[u] = xrow[idx_at(j)];
          }
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int j = j0 + u * step;
            if (j < n_o) xo_row[static_cast<int64_t>(j >> 6) * cstride + (j & 63)] = v[u];
          }
        }
      }
      for (int j = n_o + start; j < padded; j += step)
        xo_row[static_cast<int64_t>(j >> 6) * cstride + (j & 63)] = __float2half_rn(0.0f);
    }
  };
  quantise_rows(0, ncached, false);
  if (nrows > ncached) {
    __syncthreads();  // the cached rows are done: their shared memory becomes the slots
    quantise_rows(ncached, nrows, nsl > 0);
  }
  __syncthreads();   // the row cache is free from here on (phase 4 may reuse it)

  // ------------------------------------------------ phase 4: fp16 outlier slice of CB
  if (gather) {
    const int64_t chunks = (n_o + 63) >> 6;
    const int64_t nbuf = min(static_cast<int64_t>(kPrepWarps), p.cache_bytes_all / K);
    if (static_cast<int64_t>(n_o) * 64 >= K && nbuf > 0) {
      // Many outlier columns (one in 64 or more: then most 32-byte sectors of a CB row hold
      // one, and copying whole rows beats scattered byte reads -- on the OPT-175B layer with
      // 256 outlier columns the step took 3.604 ms with scattered reads, 3.566 ms with whole
      // rows): whole CB rows come by bulk copy into per-warp buffers in the
      // freed row cache -- two per warp when there is room, so that the next row's copy is
      // in flight while the warp picks this row's outlier columns -- and the warp picks the
      // columns there, lane l taking ranks 2l and 2l+1 of each chunk of 64 (one 8-byte load
      // of their indices), four chunks in flight at a time.
      const int nbw = nbuf >= 2 ? 2 : 1;            // buffers per warp
      const int nwarps = static_cast<int>(nbuf) / nbw;
      if (warp < nwarps) {
        // buffer i of this warp: shared memory at buf0 + i * boff, barrier bar0 + 8 i
        const uint32_t buf0 = smem_u32(psm) + static_cast<uint32_t>(warp * nbw * K);
        const uint32_t boff = nbw == 2 ? static_cast<uint32_t>(K) : 0u;
        const uint32_t bar0 = smem_u32(&s_rbar[warp * nbw]);
        const uint32_t boff8 = nbw == 2 ? 8u : 0u;
        uint32_t phs = 0u;  // bit i: the phase of buffer i's barrier
        const int64_t nw = static_cast<int64_t>(gridDim.x) * nwarps;
        int no_abort = 0;
        auto issue = [&](int i, int64_t row) {
          if (lane == 0) {
            // the buffer's previous reads (generic proxy) come before the copy into it
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive_expect_tx(bar0 + i * boff8, static_cast<uint32_t>(K));
            bulk_load(buf0 + i * boff, p.CB + row * K, static_cast<uint32_t>(K),
                      bar0 + i * boff8);
          }
        };
        int cur = 0;
        int64_t n = static_cast<int64_t>(blockIdx.x) * nwarps + warp;
        if (n < p.N) issue(0, n);
        const bool direct = n_o <= kPrepMaxIdx;  // every index in sidx
        for (; n < p.N; n += nw) {
          const bool more = n + nw < p.N;
          if (more && nbw == 2) issue(cur ^ 1, n + nw);
          const bool got =
              mbar_wait(bar0 + cur * boff8, (phs >> cur) & 1u, &no_abort, p.wait_limit_ns);
          phs ^= 1u << cur;
          if (!__all_sync(0xffffffffu, got)) {
            if (lane == 0) s_gfail = 1;
            if (more && nbw == 2)  // let the other copy land (bounded) before moving on
              mbar_wait(bar0 + (cur ^ 1) * boff8, (phs >> (cur ^ 1)) & 1u, &no_abort,
                        p.wait_limit_ns);
            break;
          }
          const uint8_t* rb = psm + warp * nbw * K + cur * boff;
          for (int64_t c0 = 0; c0 < chunks; c0 += 4) {
            uint32_t v0[4], v1[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int64_t j0 = (c0 + u) * 64 + 2 * lane;
              int2 jj = make_int2(0, 0);
              if (direct) {
                if (j0 < n_o) jj = *reinterpret_cast<const int2*>(sidx + j0);
              } else {
                if (j0 < n_o) jj.x = static_cast<int>(idx_at(j0));
                if (j0 + 1 < n_o) jj.y = static_cast<int>(idx_at(j0 + 1));
              }
              v0[u] = 0u;
              v1[u] = 0u;
              if (j0 < n_o) v0[u] = rb[jj.x];
              if (j0 + 1 < n_o) v1[u] = rb[jj.y];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
              if (c0 + u < chunks)
                reinterpret_cast<__half2*>(cbo + ((c0 + u) * p.N + n) * 64)[lane] =
                    codes_to_half2(v0[u], v1[u], kE4M3);
          }
          __syncwarp();
          if (nbw == 2)
            cur ^= 1;
          else if (more)
            issue(0, n + nw);
        }
      }
    } else {
      // Few outlier columns: one warp per (chunk, row) item, 8 items in flight per warp
      // (the loads are scattered bytes of CB, so latency sets the pace); the first batch
      // was loaded before phase 3.
      gather_store(first4, pv0, pv1);
      for (int64_t it0 = first4 + nw4 * U4; it0 < items4; it0 += nw4 * U4) {
        int v0[U4], v1[U4];
        gather_load(it0, v0, v1);
        gather_store(it0, v0, v1);
      }
    }
  }

  // Cache miss: the last CTA to finish its part of the slice keys the cache by this call's
  // outlier set (a CTA that gave up on a wait does not arrive, so the cache stays invalid).
  if (cmode == 2) {
    __syncthreads();
    if (tid == 0) {
      s_last = 0;
      if (!s_gfail) {
        __threadfence();
        s_last = atomicAdd(p.mask + words + 1, 1u) == gridDim.x - 1u;
      }
    }
    __syncthreads();
    if (s_last) {
      __threadfence();
      for (int64_t w = tid; w < words; w += kPrepThreads)
        __stcg(p.ocache + kOcacheHdrWords + w, smask[w]);
      __syncthreads();
      if (tid == 0) {
        const uint64_t cbp = reinterpret_cast<uint64_t>(p.CB);
        __stcg(p.ocache + 1, static_cast<uint32_t>(n_o));
        __stcg(p.ocache + 2, static_cast<uint32_t>(p.N));
        __stcg(p.ocache + 3, static_cast<uint32_t>(K));
        __stcg(p.ocache + 4, static_cast<uint32_t>(cbp));
        __stcg(p.ocache + 5, static_cast<uint32_t>(cbp >> 32));
        __threadfence();
        __stcg(p.ocache, 1u);
      }
    }
  }
}

// ====================================================================== weight quantiser
// quantize_weight_kernel: step 3 over a whole weight at the speed of HBM.  The weight is cut
// into stages of R consecutive rows (R a power of two, R * K * 2 bytes up to 32 KB); CTA b
// takes stages b, b + G, ...  Its producer thread copies each stage into a ring of
// shared-memory slots with one bulk (TMA) copy, so that several stages per SM are always
// in flight; 8 consumer warps take each row's absmax and write its codes and scale from
// shared memory: a warp per row when R >= 8, else 8 / R warps per row, combining their
// maxima through shared memory.  Two CTAs share an SM, so that one CTA's barriers and
// latencies overlap the other's work.  Codes and scales are those of quantize_rows_kernel with no
// excluded column.
constexpr int kWqWarps = 8;                            // consumer warps
constexpr int kWqThreads = (kWqWarps + 1) * 32;        // + the producer warp
constexpr int64_t kWqStageTarget = 32768;              // bytes per stage (at most)
constexpr int64_t kWqRingBytes = 98304;                // shared-memory ring (at most)
constexpr int kWqMaxSlots = 8;
constexpr int64_t kWqMaxRowBytes = 32768;              // longer rows: quantize_rows_kernel

struct WqArgs {
  const __half* W;
  int64_t N, K;
  int8_t* CB;
  float* SCB;
  bool e4m3;
  int64_t R;            // rows per stage
  int64_t stages;       // ceil(N / R)
  int slots;            // ring slots
  uint64_t wait_limit_ns;
};

__host__ __device__ inline int64_t wq_rows_per_stage(int64_t K) {
  int64_t r = 1;
  while (r < 256 && 2 * r * K * 2 <= kWqStageTarget) r *= 2;
  return r;
}

__host__ __device__ inline int wq_slots(int64_t K) {
  const int64_t stage = wq_rows_per_stage(K) * K * 2;
  const int64_t n = kWqRingBytes / stage;
  return static_cast<int>(n < kWqMaxSlots ? n : kWqMaxSlots);
}

__device__ __forceinline__ void wq_consumer_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kWqWarps * 32) : "memory");
}

// true when `v` holds in every consumer thread (a barrier of the consumer warps)
__device__ __forceinline__ bool wq_consumers_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, 1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(kWqWarps * 32)
      : "memory");
  return r != 0;
}

__global__ void __launch_bounds__(kWqThreads, 2) quantize_weight_kernel(const WqArgs a) {
  extern __shared__ __align__(128) uint8_t wsm[];
  __shared__ __align__(8) uint64_t full[kWqMaxSlots];
  __shared__ __align__(8) uint64_t empty[kWqMaxSlots];
  __shared__ float red[2][kWqWarps];
  __shared__ int abort_flag_s;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t K = a.K, R = a.R;
  const int64_t stage_bytes = R * K * 2;
  const int NS = a.slots;
  if (threadIdx.x == 0) {
    for (int i = 0; i < NS; ++i) {
      mbar_init(smem_u32(&full[i]), 1);
      mbar_init(smem_u32(&empty[i]), kWqWarps);
    }
    abort_flag_s = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = &abort_flag_s;
  const uint32_t ring = smem_u32(wsm);

  if (warp == kWqWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t issued = 0;
      bool ok = true;
      for (int64_t j = blockIdx.x; j < a.stages; j += gridDim.x, ++issued) {
        const int slot = static_cast<int>(issued % NS);
        const uint32_t ph = (issued / NS) & 1u;
        if (!mbar_wait(smem_u32(&empty[slot]), ph ^ 1u, abort_flag, a.wait_limit_ns)) {
          ok = false;
          break;
        }
        // the slot's previous reads (generic proxy) come before the copy into it
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        const int64_t r0 = j * R;
        const int64_t rows = min(R, a.N - r0);
        const uint32_t bytes = static_cast<uint32_t>(rows * K * 2);
        mbar_arrive_expect_tx(smem_u32(&full[slot]), bytes);
        bulk_load(ring + static_cast<uint32_t>(slot * stage_bytes), a.W + r0 * K, bytes,
                  smem_u32(&full[slot]));
      }
      if (!ok) {
        // wind down: the copies in flight land (bounded) before the CTA exits
        int no_abort = 0;
        const uint32_t inflight = issued < static_cast<uint32_t>(NS) ? issued : NS;
        for (uint32_t i = 0; i < inflight; ++i) {
          const uint32_t u = issued - 1 - i;
          mbar_wait(smem_u32(&full[u % NS]), (u / NS) & 1u, &no_abort, a.wait_limit_ns);
        }
      }
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int wpr = R >= kWqWarps ? 1 : static_cast<int>(kWqWarps / R);   // warps per row
  const int gpr = static_cast<int>(K / 8);                             // 16-byte groups
  const int sub = warp % wpr;
  const int start = sub * 32 + lane, step = 32 * wpr;
  const float cmax = code_max(a.e4m3);
  uint32_t it = 0;
  for (int64_t j = blockIdx.x; j < a.stages; j += gridDim.x, ++it) {
    const int slot = static_cast<int>(it % NS);
    const bool got = mbar_wait(smem_u32(&full[slot]), (it / NS) & 1u, abort_flag,
                               a.wait_limit_ns);
    // warps that share rows meet at barriers below: they must all take the same branch
    if (wpr > 1 ? !wq_consumers_all(got) : !__all_sync(0xffffffffu, got)) break;
    const int64_t r0 = j * R;
    const int64_t rows = min(R, a.N - r0);
    const uint32_t sbase = ring + static_cast<uint32_t>(slot * stage_bytes);
    // row i of the stage goes to warps i * wpr .. i * wpr + wpr - 1 (wpr > 1), or to warp
    // i % 8 (wpr == 1)
    for (int64_t i = (wpr > 1 ? warp / wpr : warp); i < (wpr > 1 ? R : rows);
         i += (wpr > 1 ? R : kWqWarps)) {
      const bool have = i < rows;
      const uint32_t rbase = sbase + static_cast<uint32_t>(i * K * 2);
      float amax = 0.0f;
      if (have) {
        float m0 = 0.0f, m1 = 0.0f;
        int v = start;
        for (; v + step < gpr; v += 2 * step) {
          m0 = fmaxf(m0, absmax8_all(lds_v4(rbase + static_cast<uint32_t>(v) * 16u)));
          m1 = fmaxf(m1, absmax8_all(lds_v4(rbase + static_cast<uint32_t>(v + step) * 16u)));
        }
        if (v < gpr) m0 = fmaxf(m0, absmax8_all(lds_v4(rbase + static_cast<uint32_t>(v) * 16u)));
        amax = warp_max(fmaxf(m0, m1));
      }
      if (wpr > 1) {
        if (lane == 0) red[it & 1u][warp] = amax;
        wq_consumer_sync();
        const int base = (warp / wpr) * wpr;
        for (int w2 = 0; w2 < wpr; ++w2) amax = fmaxf(amax, red[it & 1u][base + w2]);
      }
      if (have) {
        const float sc = amax > 0.0f ? __fdiv_rn(cmax, amax) : 0.0f;
        uint2* q = reinterpret_cast<uint2*>(a.CB + (r0 + i) * K);
        for (int v = start; v < gpr; v += step)
          q[v] = codes8_fmt(lds_v4(rbase + static_cast<uint32_t>(v) * 16u), 0u, sc, a.e4m3);
        if (sub == 0 && lane == 0) a.SCB[r0 + i] = amax;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_u32(&empty[slot]));
  }
}

// Shared-memory bytes per cached row of prepare_kernel: the row and its block maxima.
__host__ inline size_t prepare_row_bytes(int64_t K) {
  return static_cast<size_t>(K) * 2 + static_cast<size_t>((K + 127) / 128) * 4;
}

// Dynamic shared memory of prepare_kernel: a row cache of `cache_rows` rows, the mask,
// its prefix, the first kPrepMaxIdx indices, one scale per row of the CTA's block and the
// block maxima of the cached rows.
__host__ inline size_t prepare_smem_bytes(int64_t K, int64_t cache_rows, int64_t rows_per_cta) {
  const int64_t words = (K + 31) / 32;
  return static_cast<size_t>(cache_rows) * prepare_row_bytes(K) +
         static_cast<size_t>(2 * words + 2 + kPrepMaxIdx + rows_per_cta) * 4;
}

}  // namespace i8

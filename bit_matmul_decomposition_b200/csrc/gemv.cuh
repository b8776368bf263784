// gemv.cuh -- the whole layer for decode batches (T <= 16) in one kernel.  With at most
// 16 tokens each CB byte feeds at most 16 multiply-adds, so the layer is a stream of CB
// through HBM and the bound is memory bandwidth, not the tensor pipe.
//
// Source: "A Gentle Introduction to 8-bit Matrix Multiplication for transformers at
// scale" (Hugging Face blog): "LLM.int8() 的总结" (outlier columns, row-wise absmax of the
// hidden states), "内部的 MatMul" (int8 product, dequantisation by the outer product of
// the scales, fp16 product of the outlier columns); "改进范围" notes that small-batch
// inference was the slow case of the original implementation.
//
// decode_kernel: one CTA per SM; CTA b works on K-slice b % S (KS bytes of K) and on the
// 32-row tiles b / S, b / S + G, ... of CB (G CTAs per slice).  Warp roles:
//
//   producer (1 thread)  a ring of STAGES 16 KB stages filled by TMA (96 KB in flight per SM
//                        covers the HBM latency; a deeper ring only lengthens the queues
//                        every other load waits in): first (forward only)
//                        all of X in 16 KB pieces, then this slice of every row of X, then
//                        the CTA's CB tiles, 32 rows x 512 B per stage (2-D boxes of
//                        32 rows x 128 B, 128-byte swizzle: chunk j of row r lands in chunk
//                        j ^ (r % 8), so the eight rows of an ldmatrix phase hit eight
//                        different bank groups).
//   compute (8 warps)    the prologue, from the X pieces (every CTA reads all of X when it
//                        fits eight stages; otherwise the CTAs split the scan of X, combine
//                        the mask and the block maxima in global memory and meet at one
//                        grid barrier of a cooperative launch):
//                          step 1: mask bit k = some row has |x| >= threshold, and the
//                          largest |x| of every (row, 512-column block);
//                          SCx[t] = max |x| over the non-outlier columns of row t (a block
//                          free of outlier columns contributes its maximum, the others are
//                          re-read without them), the ascending outlier list;
//                          step 2 on the slice rows: Xq = round(x * fl32(127/SCx)) (half
//                          away from zero), outlier columns 0, into shared memory;
//                        then per CB stage each warp one 64-byte step of K for all 32 rows
//                        (ldmatrix of both operands, mma.sync m16n8k32 s8: two 16-row
//                        groups x 8 tokens), copying out
//                        the CB bytes of the slice's outlier columns as they pass; at a
//                        tile's end the partials go into one of EW reduction buffers
//                        (shared-memory integer adds).
//   epilogue (4 warps)   warp e drains buffer e (the CTA's tiles e, e+4, ...) into the
//                        tile's slice record in global memory,
//                          P_s[t,n] = acc_s[t,n] * SCx[t]/127 + sum_{j in slice s}
//                                     X[t,idx_j] * CB[n,idx_j]          (fp32)
//                        (the exact int32 acc_s for the raw product), and counts the
//                        arrival on the tile's counter; the CTA that completes a tile sums
//                        the S records in slice order and writes
//                          C[t,n] = fp16((sum_s P_s[t,n]) * SCB[n]/127 + bias[n]),
//                        then drops the records' lines from the L2 (discard: the records
//                        never reach DRAM; the workspace is scratch after the call).
//
// The tile counters and the words of the cooperative prologue carry the launch's epoch
// (1 .. 2^32 - 1) in their upper 32 bits.  The host clears them (one memset) before every
// launch, so no leftover bytes can carry this launch's epoch: a counter is claimed by the
// first update of the launch and plain atomics follow; mask and block-maximum words are
// tagged and updated by the same OR / max.
#pragma once

#include "common.cuh"
#include "quant.cuh"

namespace i8 {
namespace gemv {

constexpr int ROWS = 32;                    // CB rows per tile
constexpr int CW = 8;                       // compute warps
constexpr int EW = 4;                       // epilogue warps, one reduction buffer each
constexpr int PRODUCER = CW;                // warp index of the TMA producer
constexpr int EPI0 = CW + 1;                // first epilogue warp
constexpr int THREADS = (CW + 1 + EW) * 32;
constexpr int PRO_THREADS = (CW + EW) * 32;  // the warps that meet at the prologue's end
constexpr int SLICE_TARGET = 3584;          // bytes of K per slice (before rounding)
constexpr int BOXW = 128;                   // bytes of K per TMA box (one swizzle row)
constexpr int CH = 64 * CW;                 // bytes of K per stage per row
constexpr int BOXES = CH / BOXW;            // TMA boxes per stage
constexpr int STAGES = 6;
constexpr int STAGE_BYTES = ROWS * CH;      // 16 KB
constexpr int XPAD = 16;                    // xs row pitch = KS + 16 (KS % 512 == 0): the 8
                                            // token rows of an ldmatrix phase hit 8 bank groups
constexpr int RP = ROWS + 4;                // token pitch of a reduction buffer (words):
                                            // the fragment adds fall on distinct banks
constexpr int MAXO = 128;                   // outlier columns kept in shared memory
constexpr int MAXOS = 32;                   // outlier columns per slice copied from CB (the
                                            // rest are read from CB when a tile completes)
constexpr int XB = 512;                     // columns per block of the prologue's maxima
constexpr int64_t MAX_K = 65536;            // larger K take the GEMM path
constexpr int MAX_S = 32;                   // slices at MAX_K: 19
constexpr int PREFETCH = 32;                // CB stages per CTA prefetched into the L2 while
                                            // the prologue runs (~76 MB over 148 CTAs)

static_assert(CH % BOXW == 0, "whole boxes per stage");
static_assert(SLICE_TARGET % CH == 0, "slices hold whole stages");
static_assert(EW == 4, "tile i of a CTA goes to epilogue warp i % 4");
static_assert(4 * SLICE_TARGET <= STAGE_BYTES, "two slice rows of X fit one stage");
static_assert(XB == 512, "a block is 64 groups of 8 columns: two per lane");

// bytes of K per slice: K split evenly, rounded up to whole stages
__host__ __device__ inline int64_t slice_bytes(int64_t K) {
  const int64_t S = (K + SLICE_TARGET - 1) / SLICE_TARGET;
  const int64_t per = (K + S - 1) / S;
  return ((per + CH - 1) / CH) * CH;
}

__host__ __device__ inline int64_t num_slices(int64_t K) {
  const int64_t ks = slice_bytes(K);
  return (K + ks - 1) / ks;
}

// One slice record of a tile in global memory: [T][32 rows] values (a warp's access to one
// token is 128 contiguous bytes), fp32 partial outputs (forward) or int32 partial sums
// (raw product).
__host__ __device__ inline int64_t rec_bytes(int64_t T) { return T * ROWS * 4; }

__host__ __device__ inline int64_t mask_words_smem(int64_t K) {
  const int64_t a = num_slices(K) * (slice_bytes(K) / 32);
  const int64_t b = (XB / 32) * ((K + XB - 1) / XB);
  return (a > b ? a : b) + 2;
}

// Dynamic shared memory, offsets from a 1024-byte aligned base.
struct Smem {
  uint32_t ring, xs, red, cbo, mask, spre, bm, dl, rmx, idx, jinfo, xo, scx, scale, jbase, misc,
      bars, total;
};

__host__ __device__ inline uint32_t smem_take(uint32_t& off, uint64_t bytes, uint32_t align) {
  off = (off + align - 1) / align * align;
  const uint32_t o = off;
  off += static_cast<uint32_t>(bytes);
  return o;
}

__host__ __device__ inline Smem smem_layout(int NT, int64_t K) {
  Smem s;
  uint32_t off = 0;
  const int TP = NT * 8;                    // token rows held (padded)
  const int64_t KS = slice_bytes(K);
  s.ring = smem_take(off, static_cast<uint64_t>(STAGES) * STAGE_BYTES, 1024);
  s.xs = smem_take(off, static_cast<uint64_t>(TP) * (KS + XPAD), 16);
  s.red = smem_take(off, static_cast<uint64_t>(EW) * TP * RP * 4, 16);
  s.cbo = smem_take(off, static_cast<uint64_t>(EW) * MAXOS * ROWS, 16);
  s.mask = smem_take(off, static_cast<uint64_t>(mask_words_smem(K)) * 4, 16);
  s.spre = smem_take(off, static_cast<uint64_t>(KS / 32) * 4, 16);
  s.bm = smem_take(off, static_cast<uint64_t>(TP) * ((K + XB - 1) / XB) * 4, 16);
  s.dl = smem_take(off, static_cast<uint64_t>(TP) * ((K + XB - 1) / XB) * 4, 16);
  s.rmx = smem_take(off, TP * 4, 16);
  s.idx = smem_take(off, MAXO * 4, 16);
  s.jinfo = smem_take(off, MAXO * 4, 16);
  s.xo = smem_take(off, static_cast<uint64_t>(TP) * MAXO * 2, 16);
  s.scx = smem_take(off, TP * 4, 16);
  s.scale = smem_take(off, TP * 4, 16);
  s.jbase = smem_take(off, (MAX_S + 1) * 4, 16);
  s.misc = smem_take(off, 16, 16);
  s.bars = smem_take(off, (2 * STAGES + 2 * EW + 1) * 8, 16);
  s.total = off;
  return s;
}

// bytes of dynamic shared memory to request (the base is aligned up to 1024 in-kernel)
__host__ inline size_t smem_bytes(int NT, int64_t K) { return smem_layout(NT, K).total + 1024; }

struct Args {
  const __half* X;           // forward: hidden states [T, K]
  const int8_t* Xq;          // raw product (i8_igemm_s32): codes [T, K]
  int T;
  int64_t N, K;
  float thr;
  const int8_t* CB;          // [N, K] (outlier bytes beyond the copied ones are read here)
  const float* SCB;          // [N]
  const __half* bias;        // [N] or NULL
  __half* C;                 // forward output [T, N]
  int32_t* acc;              // raw output [T, N]
  uint8_t* rec;              // [n_tiles][S][T][32] slice records (fp32 or int32)
  unsigned long long* cnt;   // [n_tiles] arrival counters (epoch << 32 | arrivals)
  unsigned long long epoch;  // this launch's epoch, 1 .. 2^32 - 1
  uint64_t lim;              // bound of every wait, ns
  // cooperative prologue (larger X): the CTAs split the scan of X and meet at one grid
  // barrier; the words carry the epoch in their upper 32 bits and start at zero
  bool coop;
  unsigned long long* gmask;  // [ceil(K/32)] outlier mask words
  unsigned long long* gbm;    // [T][ceil(K/512)] block keys (largest |x| below the
                              // threshold and its column, as block_key8 packs them)
  unsigned long long* gbar;   // [1] barrier counter (epoch << 32 | arrivals)
};

__device__ __forceinline__ void mma_s8_16816(int (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                             uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+r"(c[0]), "+r"(c[1]), "+r"(c[2]), "+r"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Prefetch one box of CB into the L2 (no shared memory, no completion to wait for).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap* m, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"(
                   reinterpret_cast<uint64_t>(m)),
               "r"(x), "r"(y)
               : "memory");
}

// Four 8 x 16-byte matrices from shared memory (lane l gives the address of row l % 8 of
// matrix l / 8); lane l receives bytes 4 (l % 4) .. 4 (l % 4) + 3 of row l / 4 of each.
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t lds_u8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ void all_sync() {   // compute + epilogue warps
  asm volatile("bar.sync 1, %0;" ::"n"(PRO_THREADS) : "memory");
}

__device__ __forceinline__ void compute_sync() {   // compute warps
  asm volatile("bar.sync 2, %0;" ::"n"(CW * 32) : "memory");
}

__device__ __forceinline__ void fence_acq_rel_gpu() {
  asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

// max |x| of 8 fp16 values as the bit pattern of the fp16 absolute value (the patterns of
// non-negative fp16 numbers order like the numbers)
__device__ __forceinline__ uint32_t absmax8_bits(const uint4 v) {
  const __half2 a = __habs2(*reinterpret_cast<const __half2*>(&v.x));
  const __half2 b = __habs2(*reinterpret_cast<const __half2*>(&v.y));
  const __half2 c = __habs2(*reinterpret_cast<const __half2*>(&v.z));
  const __half2 d = __habs2(*reinterpret_cast<const __half2*>(&v.w));
  const __half2 m = __hmax2(__hmax2(a, b), __hmax2(c, d));
  const uint32_t u = *reinterpret_cast<const uint32_t*>(&m);
  const uint32_t lo = u & 0xffffu, hi = u >> 16;
  return lo > hi ? lo : hi;
}

__device__ __forceinline__ float half_bits_to_float(uint32_t b) {
  return __half2float(__ushort_as_half(static_cast<unsigned short>(b)));
}

// Block key of 8 fp16 values at columns c0 .. c0 + 7 of a 512-column block: the largest
// |x| among the values not in `skip`, as its fp16 bit pattern, in the upper 16 bits, and its
// column within the block in the lower ones (the larger column on ties); 0 when every value
// is skipped.  The unsigned maximum of keys is the key of their union.
__device__ __forceinline__ uint32_t block_key8(const uint4 v, uint32_t c0, uint32_t skip) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t key = 0u;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t k0 = ((w[i] & 0x7fffu) << 16) | (c0 + 2 * i);
    const uint32_t k1 = (w[i] & 0x7fff0000u) | (c0 + 2 * i + 1);
    if (!((skip >> (2 * i)) & 1u)) key = max(key, k0);
    if (!((skip >> (2 * i + 1)) & 1u)) key = max(key, k1);
  }
  return key;
}

// The block key of a group of 8 values over those below the threshold; their outlier bits
// (|x| >= thr) go to *bits.
__device__ __forceinline__ uint32_t group_key(const uint4 v, uint32_t c0, float thr,
                                              uint32_t* bits) {
  uint32_t key = block_key8(v, c0, 0u);
  *bits = 0u;
  if (half_bits_to_float(key >> 16) >= thr) {   // rare: a value at the threshold
    *bits = outlier_bits8(v, thr);
    key = block_key8(v, c0, *bits);
  }
  return key;
}

// Epoch-tagged words: the upper 32 bits hold the epoch of the launch that last claimed the
// word, and a word of another epoch reads as zero.  The first update in a launch claims
// the word with one compare-and-swap (a late claim finds it changed and fails harmlessly),
// after which plain atomics apply -- no retry loops, however many CTAs update it.
__device__ __forceinline__ void tag_claim(unsigned long long* w, uint32_t e) {
  const unsigned long long v = __ldcg(w);
  if (static_cast<uint32_t>(v >> 32) != e) atomicCAS(w, v, static_cast<unsigned long long>(e) << 32);
}

__device__ __forceinline__ uint32_t tagged_get(const unsigned long long* w, uint32_t e) {
  const unsigned long long v = __ldcg(w);
  return static_cast<uint32_t>(v >> 32) == e ? static_cast<uint32_t>(v) : 0u;
}

// Arrival on a tile counter: the number of arrivals of this epoch including this one.
__device__ __forceinline__ int tile_arrive(unsigned long long* c, uint32_t e) {
  tag_claim(c, e);
  return static_cast<int>(static_cast<uint32_t>(atomicAdd(c, 1ull))) + 1;
}

// Grid barrier of the cooperative launch (one thread per CTA), in two halves so that
// independent work can go between them.  The counter only grows within an epoch (a replay
// of the same launch starts the next generation of `target` arrivals).  The wait is
// bounded: false after `lim` ns (the error word records it).
__device__ __forceinline__ uint32_t grid_arrive(unsigned long long* ctr, uint32_t e,
                                                uint32_t target, bool claimed = false) {
  fence_acq_rel_gpu();  // this CTA's writes before its arrival
  if (!claimed) tag_claim(ctr, e);
  const uint32_t c = static_cast<uint32_t>(atomicAdd(ctr, 1ull));
  return (c / target + 1) * target;
}

__device__ __forceinline__ bool grid_wait(unsigned long long* ctr, uint32_t e, uint32_t goal,
                                          uint64_t lim) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 0;; ++it) {
    const unsigned long long v = __ldcg(ctr);
    if (static_cast<uint32_t>(v >> 32) == e && static_cast<uint32_t>(v) >= goal) break;
    if ((it & 15u) == 15u && globaltimer_ns() - t0 > lim) {
      raise_error(kErrWaitTimeout);
      return false;
    }
  }
  fence_acq_rel_gpu();
  return true;
}

__device__ __forceinline__ bool grid_sync(unsigned long long* ctr, uint32_t e, uint32_t target,
                                          uint64_t lim, bool claimed = false) {
  return grid_wait(ctr, e, grid_arrive(ctr, e, target, claimed), lim);
}

// Consumer side of the ring: wait for stage s (phase ph), then advance.
struct Ring {
  uint32_t full, empty;  // shared addresses of the first full / empty barrier
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ uint32_t full_bar() const { return full + 8u * s; }
  __device__ __forceinline__ uint32_t empty_bar() const { return empty + 8u * s; }
  __device__ __forceinline__ void advance() {
    if (++s == STAGES) {
      s = 0;
      ph ^= 1u;
    }
  }
};

// ---------------------------------------------------------------------- forward prologue
// Run by the compute warps (ct = thread index among them).  Consumes the X stages of the
// ring in the producer's order: (unless a.coop) the ceil(2TK / STAGE_BYTES) pieces of the
// flat X starting at piece blockIdx.x (mod their count), then the T slice rows starting at
// row blockIdx.x / S (mod T) -- the CTAs start at different places, which spreads their
// reads of X over the L2 slices.  Leaves the slice of Xq in xs, the mask, ranks, SCx and
// the outlier tables in shared memory.  Returns false when a wait gave up.
template <int NT>
__device__ __forceinline__ bool forward_prologue(
    const Args& a, const int ct, const int slice, const int64_t KS, const int S, Ring& rg,
    const uint8_t* ring_p, uint8_t* xs, const int64_t pitch, uint32_t* maskall, int32_t* spre,
    uint32_t* bm, int32_t* dl, uint32_t* rmx, int32_t* idx_s, uint32_t* jinfo, __half* xo_s,
    float* scx, float* scale, int32_t* jbase, int* misc, uint64_t* xq_bar,
    volatile int* abort_flag) {
  const int T = a.T;
  const int64_t K = a.K;
  const __half* __restrict__ X = a.X;
  const float thr = a.thr;
  const int64_t KW = (K + 31) / 32;
  const int64_t NBK = (K + XB - 1) / XB;
  const int64_t G = K / 8;  // 16-byte groups of 8 columns per row
  const int w = ct >> 5, lane = ct & 31;
  constexpr int GPB = XB / 8;  // groups per block

  bool ok = true;
  const uint32_t e = static_cast<uint32_t>(a.epoch);
  // One row: a column is an outlier column exactly when its one element reaches the
  // threshold, so the row maximum over the other columns is the largest |x| below the
  // threshold, taken in the same pass as the mask (no block maxima, no re-read).
  const bool one_row = (T == 1);
  if (!a.coop) {
    // (a) step 1 and the block maxima (one row: the row maximum), piece by piece
    const int64_t xbytes = static_cast<int64_t>(T) * K * 2;
    const int64_t pieces = (xbytes + STAGE_BYTES - 1) / STAGE_BYTES;
    for (int64_t pc = 0; pc < pieces; ++pc) {
      if (ok) {
        const bool got = mbar_wait(rg.full_bar(), rg.ph, abort_flag, a.lim);
        ok = __all_sync(0xffffffffu, got);
      }
      if (ok) {
        const int p = static_cast<int>((pc + blockIdx.x) % pieces);
        const uint4* sp = reinterpret_cast<const uint4*>(ring_p + rg.s * STAGE_BYTES);
        const int64_t left = xbytes - static_cast<int64_t>(p) * STAGE_BYTES;
        const int nvec = static_cast<int>(min(static_cast<int64_t>(STAGE_BYTES), left) / 16);
        const int Gi = static_cast<int>(G);
        if ((Gi & 31) == 0) {
          // the 32 groups of a warp lie in one row and one block (rows are whole multiples
          // of 32 groups, blocks of 64)
          for (int i0 = w * 32; i0 < nvec; i0 += CW * 32) {
            const int f0 = p * (STAGE_BYTES / 16) + i0;  // flat group index of lane 0
            const int t = f0 / Gi;
            const int g = f0 - t * Gi + lane;
            const uint4 v = sp[i0 + lane];
            uint32_t bits;
            const uint32_t key =
                group_key(v, static_cast<uint32_t>((g & (GPB - 1)) * 8), thr, &bits);
            if (bits) atomicOr(&maskall[g >> 2], bits << (8 * (g & 3)));
            const uint32_t mx = __reduce_max_sync(0xffffffffu, key);
            if (lane == 0) {
              if (one_row)   // the largest |x| below the threshold
                atomicMax(&rmx[0], __float_as_uint(half_bits_to_float(mx >> 16)));
              else
                atomicMax(&bm[t * NBK + g / GPB], mx);
            }
          }
        } else {
          for (int i0 = w * 32; i0 < nvec; i0 += CW * 32) {
            const int i = i0 + lane;
            const bool valid = i < nvec;
            uint32_t m = 0u, key = 0xffffffffu;
            if (valid) {
              const uint4 v = sp[i];
              const int gf = p * (STAGE_BYTES / 16) + i;  // group index in the flat X
              const int t = gf / Gi, g = gf - t * Gi;
              uint32_t bits;
              m = group_key(v, static_cast<uint32_t>((g & (GPB - 1)) * 8), thr, &bits);
              if (bits) atomicOr(&maskall[g >> 2], bits << (8 * (g & 3)));
              key = one_row ? 0u : static_cast<uint32_t>(t * NBK + g / GPB);
            }
            const uint32_t peers = __match_any_sync(0xffffffffu, key);
            const uint32_t mx = __reduce_max_sync(peers, m);
            if (valid && lane == __ffs(peers) - 1) {
              if (one_row)
                atomicMax(&rmx[0], __float_as_uint(half_bits_to_float(mx >> 16)));
              else
                atomicMax(&bm[key], mx);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(rg.empty_bar());
      }
      rg.advance();
    }
    compute_sync();

  } else {
    // (a') the CTAs split X into shares of 16-byte groups.  Each ORs the outlier bits of its
    // share into the global mask and takes the maxima of its share into the global block
    // maxima (words that start at zero: an OR or max with the epoch in the upper half both
    // tags and updates them); one grid barrier; then every CTA copies the final mask and
    // block maxima into shared memory, where they stand exactly as if the CTA had scanned
    // all of X itself, and the rest of the prologue is the same for both paths.
    const int64_t TG = static_cast<int64_t>(T) * G;
    const int64_t f_lo = TG * blockIdx.x / gridDim.x, f_hi = TG * (blockIdx.x + 1) / gridDim.x;
    const unsigned long long eh = static_cast<unsigned long long>(e) << 32;
    if (ct == 0) tag_claim(a.gbar, e);   // while the scan's loads are in flight
    for (int64_t f0 = f_lo + w * 32; f0 < f_hi; f0 += CW * 32) {
      const int64_t f = f0 + lane;
      const bool valid = f < f_hi;
      uint32_t m = 0u, key = 0xffffffffu;
      if (valid) {
        const int64_t t = f / G, g = f - t * G;
        const uint4 v = ldg_v4(X + t * K + g * 8);
        uint32_t bits;
        m = group_key(v, static_cast<uint32_t>((g & (GPB - 1)) * 8), thr, &bits);
        if (bits) atomicOr(a.gmask + (g >> 2), eh | (bits << (8 * (g & 3))));
        key = static_cast<uint32_t>(t * NBK + g / GPB);
      }
      const uint32_t peers = __match_any_sync(0xffffffffu, key);
      const uint32_t mx = __reduce_max_sync(peers, m);
      if (valid && lane == __ffs(peers) - 1) atomicMax(a.gbm + key, eh | mx);
    }
    compute_sync();
    if (ct == 0 && !grid_sync(a.gbar, e, gridDim.x, a.lim, true)) *abort_flag = 1;
    compute_sync();
    ok = *abort_flag == 0;
    for (int64_t x = ct; x < KW; x += CW * 32) maskall[x] = ok ? tagged_get(a.gmask + x, e) : 0u;
    for (int64_t i = ct; i < static_cast<int64_t>(T) * NBK; i += CW * 32)
      bm[i] = ok ? tagged_get(a.gbm + i, e) : 0u;
    compute_sync();
  }

  // (b) ranks: the compute threads take contiguous runs of mask words, and one block-wide
  // exclusive scan of the runs' outlier counts gives each word its rank base
  const int WPS = static_cast<int>(KS / 32);  // mask words per slice
  {
    const int KWi = static_cast<int>(KW);
    const int cw = (KWi + CW * 32 - 1) / (CW * 32);
    const int wb = ct * cw < KWi ? ct * cw : KWi;
    const int we = wb + cw < KWi ? wb + cw : KWi;
    int cnt = 0;
    for (int x = wb; x < we; ++x) cnt += __popc(maskall[x]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    int* wsum = reinterpret_cast<int*>(jinfo);  // scratch until (c) fills jinfo
    if (lane == 31) wsum[w] = incl;
    compute_sync();
    int before = 0, total = 0;
#pragma unroll
    for (int i = 0; i < CW; ++i) {
      const int v = wsum[i];
      before += i < w ? v : 0;
      total += v;
    }
    int run = before + incl - cnt;
    const int sw0 = slice * WPS;
    for (int x = wb; x < we; ++x) {
      if (x % WPS == 0) jbase[x / WPS] = run;
      if (x >= sw0 && x < sw0 + WPS) spre[x - sw0] = run;
      uint32_t bits = maskall[x];
      while (bits) {
        const int bpos = __ffs(bits) - 1;
        bits &= bits - 1u;
        if (run < MAXO) idx_s[run] = x * 32 + bpos;
        ++run;
      }
    }
    if (ct == 0) {
      misc[0] = total;  // n_o
      jbase[S] = total;
    }
  }
  compute_sync();

  // (c) the row scales, where each kept outlier column is found in the epilogue, and its
  // X values
  const int n_o = misc[0];
  const int nf = n_o < MAXO ? n_o : MAXO;
  // jinfo[j]: 0 when the CTAs of column idx_j's slice copy its CB bytes (rank below MAXOS
  // in the slice), else 0x80000000 | idx_j (read from CB when the tile completes)
  for (int j = ct; j < nf; j += CW * 32) {
    const int c = idx_s[j];
    const int jl = j - jbase[c / static_cast<int>(KS)];
    jinfo[j] = jl < MAXOS ? 0u : (0x80000000u | static_cast<uint32_t>(c));
  }
  for (int i = ct; i < T * nf; i += CW * 32) {
    const int t = i / nf, j = i - t * nf;
    xo_s[t * MAXO + j] = X[static_cast<int64_t>(t) * K + idx_s[j]];
  }
  if (!one_row) {
    // Row maxima from the block keys: a block free of outlier columns, or one whose largest
    // value below the threshold lies in a column that is not an outlier column, gives that
    // value; the remaining (row, block) pairs are listed and re-read from X without the
    // outlier columns.  (With systematic outlier columns -- large in every row -- the list
    // stays empty.)
    if (ct == 0) misc[2] = 0;
    compute_sync();
    for (int t = w; t < T; t += CW) {
      uint32_t m = 0u;
      for (int64_t b0 = 0; b0 < NBK; b0 += 32) {
        const int64_t b = b0 + lane;
        if (b < NBK) {
          uint32_t o = 0u;
#pragma unroll
          for (int i = 0; i < XB / 32; ++i) o |= maskall[b * (XB / 32) + i];
          const uint32_t key = bm[t * NBK + b];
          const int64_t col = b * XB + (key & 0xffffu);
          if (o == 0u || !((maskall[col >> 5] >> (col & 31)) & 1u))
            m = max(m, key >> 16);
          else
            dl[atomicAdd(&misc[2], 1)] = static_cast<int32_t>(t * NBK + b);
        }
      }
      m = __reduce_max_sync(0xffffffffu, m);
      if (lane == 0) rmx[t] = __float_as_uint(half_bits_to_float(m));
    }
    compute_sync();
    // the listed pairs, re-read without the outlier columns: a warp takes pairs, two groups
    // of 8 columns per lane, four pairs' loads in flight
    {
      const int pairs = misc[2];
      constexpr int U = 4;
      for (int q0 = w; q0 < pairs; q0 += CW * U) {
        uint4 v[U][2];
        uint32_t sk[U][2];
        int tt[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const int q = q0 + u * CW;
          tt[u] = 0;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            v[u][h] = make_uint4(0u, 0u, 0u, 0u);
            sk[u][h] = 0xffu;
          }
          if (q < pairs) {
            const int pr = dl[q];
            const int t = static_cast<int>(pr / NBK), d = static_cast<int>(pr - t * NBK);
            tt[u] = t;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int64_t g = static_cast<int64_t>(d) * GPB + h * 32 + lane;
              if (g < G) {
                v[u][h] = ldg_v4(X + static_cast<int64_t>(t) * K + g * 8);
                sk[u][h] = (maskall[g >> 2] >> (8 * (g & 3))) & 0xffu;
              }
            }
          }
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
          if (q0 + u * CW < pairs) {  // uniform over the warp
            const float m = fmaxf(absmax8(v[u][0], sk[u][0]), absmax8(v[u][1], sk[u][1]));
            const uint32_t mm = __reduce_max_sync(0xffffffffu, __float_as_uint(m));
            if (lane == 0) atomicMax(&rmx[tt[u]], mm);
          }
        }
      }
    }
  }
  compute_sync();
  for (int t = ct; t < T; t += CW * 32) {
    const float m = __uint_as_float(rmx[t]);
    scx[t] = m;
    scale[t] = m > 0.0f ? __fdiv_rn(127.0f, m) : 0.0f;
  }
  compute_sync();

  // (d) step 2 on this slice: two rows of X per ring stage, in the producer's order
  {
    const int64_t k0 = static_cast<int64_t>(slice) * KS;
    const int64_t klen = KS < K - k0 ? KS : K - k0;
    const int64_t gl = klen / 8;
    for (int i = 0; i < T; i += 2) {
      if (ok) {
        const bool got = mbar_wait(rg.full_bar(), rg.ph, abort_flag, a.lim);
        ok = __all_sync(0xffffffffu, got);
      }
      if (ok) {
        for (int h = 0; h < 2 && i + h < T; ++h) {
          const int t = static_cast<int>((i + h + blockIdx.x / S) % T);
          const uint4* sp =
              reinterpret_cast<const uint4*>(ring_p + rg.s * STAGE_BYTES + h * klen * 2);
          const float sc = scale[t];
          for (int64_t q = ct; q < gl; q += CW * 32) {
            const int64_t g = k0 / 8 + q;
            const uint32_t skip = (maskall[g >> 2] >> (8 * (g & 3))) & 0xffu;
            *reinterpret_cast<uint2*>(xs + t * pitch + q * 8) = codes8(sp[q], skip, sc);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(rg.empty_bar());
      }
      rg.advance();
    }
  }
  return ok;
}

// ---------------------------------------------------------------------- tile completion
// Run by the epilogue warp of the CTA whose arrival completed `tile`: sums the S slice
// records in slice order and writes the raw int32 sums (kRaw) or the fp16 output, adding
// the outlier columns whose CB bytes no slice copied.  Lane r owns output channel
// tile * 32 + r, all tokens.
template <int NT, bool kRaw>
__device__ __forceinline__ void finish_tile(const Args& a, const int64_t tile, const int S,
                                            const int rb, const uint32_t* maskall,
                                            const int32_t* idx_s, const uint32_t* jinfo,
                                            const __half* xo_s, const int* misc) {
  constexpr int TP = NT * 8;
  const int lane = threadIdx.x & 31;
  const int T = a.T;
  const int64_t N = a.N, K = a.K;
  const int64_t n = tile * ROWS + lane;
  const uint8_t* tb = a.rec + tile * S * rb + lane * 4;  // this row in slice 0's record
  if constexpr (kRaw) {
    int32_t acc[TP];
#pragma unroll
    for (int t = 0; t < TP; ++t) acc[t] = 0;
    for (int sp = 0; sp < S; sp += 2) {  // two records' loads in flight at a time
      const int32_t* p0 = reinterpret_cast<const int32_t*>(tb + static_cast<int64_t>(sp) * rb);
      const int32_t* p1 = reinterpret_cast<const int32_t*>(tb + static_cast<int64_t>(sp + 1) * rb);
      const bool two = sp + 1 < S;
      int32_t v0[TP], v1[TP];
#pragma unroll
      for (int t = 0; t < TP; ++t) {
        v0[t] = t < T ? __ldcg(p0 + t * ROWS) : 0;
        v1[t] = (two && t < T) ? __ldcg(p1 + t * ROWS) : 0;
      }
#pragma unroll
      for (int t = 0; t < TP; ++t) acc[t] += v0[t] + v1[t];
    }
    if (n < N) {
#pragma unroll
      for (int t = 0; t < TP; ++t)
        if (t < T) a.acc[static_cast<int64_t>(t) * N + n] = acc[t];
    }
  } else {
    float ws = 0.0f, bn = 0.0f;
    if (n < N) {
      ws = __ldg(a.SCB + n) * (1.0f / 127.0f);
      bn = a.bias ? __half2float(a.bias[n]) : 0.0f;
    }
    float part[TP];
#pragma unroll
    for (int t = 0; t < TP; ++t) part[t] = 0.0f;
    for (int sp = 0; sp < S; sp += 2) {
      const float* p0 = reinterpret_cast<const float*>(tb + static_cast<int64_t>(sp) * rb);
      const float* p1 = reinterpret_cast<const float*>(tb + static_cast<int64_t>(sp + 1) * rb);
      const bool two = sp + 1 < S;
      float v0[TP], v1[TP];
#pragma unroll
      for (int t = 0; t < TP; ++t) {
        v0[t] = t < T ? __ldcg(p0 + t * ROWS) : 0.0f;
        v1[t] = (two && t < T) ? __ldcg(p1 + t * ROWS) : 0.0f;
      }
#pragma unroll
      for (int t = 0; t < TP; ++t) part[t] = (part[t] + v0[t]) + v1[t];
    }
    // outlier columns whose CB bytes were not copied: the first MAXO through jinfo, the
    // rest by walking the mask from the column after the last kept index
    const int n_o = misc[0];
    const int nf = n_o < MAXO ? n_o : MAXO;
    for (int j = 0; j < nf; ++j) {
      const uint32_t inf = jinfo[j];
      if (inf != 0u) {
        const float cb =
            n < N ? static_cast<float>(__ldg(a.CB + n * K + (inf & 0x7fffffffu))) : 0.0f;
#pragma unroll
        for (int t = 0; t < TP; ++t)
          if (t < T) part[t] = fmaf(__half2float(xo_s[t * MAXO + j]), cb, part[t]);
      }
    }
    if (n_o > MAXO) {
      const int64_t KW = (K + 31) / 32;
      const int c0 = idx_s[MAXO - 1];
      int64_t w = c0 >> 5;
      uint32_t bits = (c0 & 31) == 31 ? 0u : (maskall[w] & ~((2u << (c0 & 31)) - 1u));
      while (true) {
        while (bits == 0u && w + 1 < KW) bits = maskall[++w];
        if (bits == 0u) break;
        const int bp = __ffs(bits) - 1;
        bits &= bits - 1u;
        const int64_t col = w * 32 + bp;
        const float cb = n < N ? static_cast<float>(__ldg(a.CB + n * K + col)) : 0.0f;
#pragma unroll
        for (int t = 0; t < TP; ++t)
          if (t < T)
            part[t] = fmaf(__half2float(a.X[static_cast<int64_t>(t) * K + col]), cb, part[t]);
      }
    }
    if (n < N) {
#pragma unroll
      for (int t = 0; t < TP; ++t)
        if (t < T) a.C[static_cast<int64_t>(t) * N + n] = __float2half_rn(fmaf(part[t], ws, bn));
    }
  }
  // The S records are summed (every loaded value has reached the stores above): drop their
  // L2 lines so they are never written back to DRAM.  Only whole 128-byte lines inside
  // this tile's records are dropped.
  __syncwarp();
  const uintptr_t lo = reinterpret_cast<uintptr_t>(a.rec + tile * S * rb);
  const uintptr_t hi = lo + static_cast<uintptr_t>(S) * static_cast<uintptr_t>(rb);
  for (uintptr_t p = ((lo + 127u) & ~static_cast<uintptr_t>(127u)) + lane * 128u; p + 128u <= hi;
       p += 32u * 128u)
    asm volatile("discard.global.L2 [%0], 128;" ::"l"(p) : "memory");
}

// ---------------------------------------------------------------------- the kernel
// kRaw: the int8 product of given codes (a.Xq) written as int32 (a.acc); otherwise the
// forward from a.X to a.C.  Launched with one CTA per SM, a multiple of S CTAs.
template <int NT, bool kRaw>
__global__ void __launch_bounds__(THREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmCB, const Args a) {
  constexpr int TP = NT * 8;
  extern __shared__ uint8_t smraw[];
  const uint32_t raw_s = smem_u32(smraw);
  const uint32_t pad = (1024u - (raw_s & 1023u)) & 1023u;
  uint8_t* sm = smraw + pad;
  const int T = a.T;
  const int64_t N = a.N, K = a.K;
  const Smem L = smem_layout(NT, K);
  const int64_t KS = slice_bytes(K);
  const int S = static_cast<int>(num_slices(K));
  const int64_t pitch = KS + XPAD;
  const uint32_t ring = raw_s + pad + L.ring;
  const uint8_t* ring_p = sm + L.ring;
  uint8_t* xs = sm + L.xs;
  int32_t* red = reinterpret_cast<int32_t*>(sm + L.red);
  uint8_t* cbo = sm + L.cbo;
  uint32_t* maskall = reinterpret_cast<uint32_t*>(sm + L.mask);
  int32_t* spre = reinterpret_cast<int32_t*>(sm + L.spre);
  uint32_t* bm = reinterpret_cast<uint32_t*>(sm + L.bm);
  int32_t* dl = reinterpret_cast<int32_t*>(sm + L.dl);
  uint32_t* rmx = reinterpret_cast<uint32_t*>(sm + L.rmx);
  int32_t* idx_s = reinterpret_cast<int32_t*>(sm + L.idx);
  uint32_t* jinfo = reinterpret_cast<uint32_t*>(sm + L.jinfo);
  __half* xo_s = reinterpret_cast<__half*>(sm + L.xo);
  float* scx = reinterpret_cast<float*>(sm + L.scx);
  float* scale = reinterpret_cast<float*>(sm + L.scale);
  int32_t* jbase = reinterpret_cast<int32_t*>(sm + L.jbase);
  int* misc = reinterpret_cast<int*>(sm + L.misc);  // [0] n_o, [1] abort flag, [2] scratch
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + L.bars);
  uint64_t* empty = full + STAGES;
  uint64_t* rfull = empty + STAGES;
  uint64_t* rempty = rfull + EW;
  uint64_t* xq_bar = rempty + EW;  // raw mode: the code rows have landed in xs

  const int slice = static_cast<int>(blockIdx.x % S);
  const int cta_in_slice = static_cast<int>(blockIdx.x / S);
  const int ctas_in_slice = (static_cast<int>(gridDim.x) - slice + S - 1) / S;
  const int64_t k0 = static_cast<int64_t>(slice) * KS;
  const int64_t klen = KS < K - k0 ? KS : K - k0;
  const int spt = static_cast<int>((klen + CH - 1) / CH);  // stages per tile
  const int64_t n_tiles = (N + ROWS - 1) / ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(smem_u32(full + i), 1);
      mbar_init(smem_u32(empty + i), CW);
    }
    for (int i = 0; i < EW; ++i) {
      mbar_init(smem_u32(rfull + i), CW);
      mbar_init(smem_u32(rempty + i), 1);
    }
    mbar_init(smem_u32(xq_bar), 1);
    misc[0] = 0;
    misc[1] = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort_flag = misc + 1;

  if (warp == PRODUCER) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      tma_prefetch_desc(&tmCB);
      int s = 0;
      uint32_t ph = 0;
      uint32_t issued = 0;
      bool ok = true;
      // one ring stage per copy: wait until it is free, arm it, return its full barrier
      auto acquire = [&](uint32_t bytes) -> uint32_t {
        if (!mbar_wait(smem_u32(empty + s), ph ^ 1u, abort_flag, a.lim)) return 0u;
        const uint32_t fb = smem_u32(full + s);
        mbar_arrive_expect_tx(fb, bytes);
        return fb;
      };
      auto advance = [&]() {
        ++issued;
        if (++s == STAGES) {
          s = 0;
          ph ^= 1u;
        }
      };
      grid_dep_wait();  // X (or the codes) may come from the previous kernel
      if constexpr (kRaw) {
        // this slice of the code rows straight into xs
        mbar_arrive_expect_tx(smem_u32(xq_bar), static_cast<uint32_t>(T * klen));
        for (int t = 0; t < T; ++t)
          bulk_load(smem_u32(xs + t * pitch), a.Xq + static_cast<int64_t>(t) * K + k0,
                    static_cast<uint32_t>(klen), smem_u32(xq_bar));
      } else {
        const uint8_t* xb = reinterpret_cast<const uint8_t*>(a.X);
        const int64_t xbytes = static_cast<int64_t>(T) * K * 2;
        const int64_t pieces = a.coop ? 0 : (xbytes + STAGE_BYTES - 1) / STAGE_BYTES;
        for (int64_t pc = 0; pc < pieces && ok; ++pc) {
          const int64_t off = ((pc + blockIdx.x) % pieces) * STAGE_BYTES;
          const uint32_t bytes =
              static_cast<uint32_t>(min(static_cast<int64_t>(STAGE_BYTES), xbytes - off));
          const uint32_t fb = acquire(bytes);
          if (!fb) {
            ok = false;
            break;
          }
          bulk_load(ring + s * STAGE_BYTES, xb + off, bytes, fb);
          advance();
        }
        // this slice of the rows of X, two rows per stage (rows (i + cta_in_slice) % T in
        // order of i); once the ring is full, the CTA's first CB stages are prefetched into
        // the L2, so that HBM streams CB while the prologue runs
        bool prefetched = false;
        auto prefetch_cb = [&]() {
          prefetched = true;
          int n = 0;
          for (int64_t tile = cta_in_slice; tile < n_tiles && n < PREFETCH;
               tile += ctas_in_slice) {
            for (int st = 0; st < spt && n < PREFETCH; ++st, ++n) {
              const int x = static_cast<int>(k0 + static_cast<int64_t>(st) * CH);
#pragma unroll
              for (int c = 0; c < BOXES; ++c)
                tma_prefetch_l2_2d(&tmCB, x + c * BOXW, static_cast<int>(tile * ROWS));
            }
          }
        };
        const uint32_t rb = static_cast<uint32_t>(klen * 2);
        for (int i = 0; i < T && ok; i += 2) {
          if (!prefetched && issued >= static_cast<uint32_t>(STAGES)) prefetch_cb();
          const int ta = (i + cta_in_slice) % T;
          const int tb = (i + 1 + cta_in_slice) % T;
          const bool two = i + 1 < T;
          const uint32_t fb = acquire(two ? 2 * rb : rb);
          if (!fb) {
            ok = false;
            break;
          }
          bulk_load(ring + s * STAGE_BYTES, xb + (static_cast<int64_t>(ta) * K + k0) * 2, rb, fb);
          if (two)
            bulk_load(ring + s * STAGE_BYTES + rb, xb + (static_cast<int64_t>(tb) * K + k0) * 2,
                      rb, fb);
          advance();
        }
        if (!prefetched && ok) prefetch_cb();
      }
      for (int64_t tile = cta_in_slice; tile < n_tiles && ok; tile += ctas_in_slice) {
        const int y = static_cast<int>(tile * ROWS);
        for (int st = 0; st < spt; ++st) {
          const uint32_t fb = acquire(STAGE_BYTES);
          if (!fb) {
            ok = false;
            break;
          }
          const int x = static_cast<int>(k0 + static_cast<int64_t>(st) * CH);
#pragma unroll
          for (int c = 0; c < BOXES; ++c)
            tma_load_2d(ring + s * STAGE_BYTES + c * (ROWS * BOXW), &tmCB, fb, x + c * BOXW, y);
          advance();
        }
      }
      if (!ok) {
        // wind down: let the copies in flight land (bounded) before the CTA exits
        int no_abort = 0;
        const uint32_t inflight = issued < STAGES ? issued : STAGES;
        for (uint32_t i = 0; i < inflight; ++i) {
          const uint32_t u = issued - 1 - i;
          mbar_wait(smem_u32(full + u % STAGES), (u / STAGES) & 1u, &no_abort, a.lim);
        }
      }
      if constexpr (kRaw) {
        int no_abort = 0;  // the code rows must land before the CTA may exit
        mbar_wait(smem_u32(xq_bar), 0u, &no_abort, a.lim);
      }
    }
  } else {
    const int pt = warp < PRODUCER ? threadIdx.x : threadIdx.x - 32;
    // zero the reduction buffers, (forward) the mask and block maxima, and every byte of
    // xs that no code row writes: rows >= T, and columns >= klen of the others
    for (int i = pt; i < EW * TP * RP; i += PRO_THREADS) red[i] = 0;
    if constexpr (!kRaw) {
      const int64_t MW = mask_words_smem(K), nbm = TP * ((K + XB - 1) / XB);
      for (int64_t i = pt; i < MW; i += PRO_THREADS) maskall[i] = 0u;
      for (int64_t i = pt; i < nbm; i += PRO_THREADS) bm[i] = 0u;
      for (int i = pt; i < TP; i += PRO_THREADS) rmx[i] = 0u;
    }
    {
      const int64_t tail = (pitch - klen) / 16, per_row = pitch / 16;
      for (int64_t i = pt; i < T * tail; i += PRO_THREADS) {
        const int64_t t = i / tail, c = i - t * tail;
        *reinterpret_cast<uint4*>(xs + t * pitch + klen + c * 16) = make_uint4(0u, 0u, 0u, 0u);
      }
      for (int64_t i = pt; i < (TP - T) * per_row; i += PRO_THREADS)
        reinterpret_cast<uint4*>(xs + T * pitch)[i] = make_uint4(0u, 0u, 0u, 0u);
    }
    all_sync();
    Ring rg;
    rg.full = smem_u32(full);
    rg.empty = smem_u32(empty);
    bool ok = true;
    if (warp < CW) {
      if constexpr (kRaw) {
        const bool got = mbar_wait(smem_u32(xq_bar), 0u, abort_flag, a.lim);
        ok = __all_sync(0xffffffffu, got);
      } else {
        grid_dep_wait();  // the prologue re-reads a few blocks of X from global memory
        ok = forward_prologue<NT>(a, threadIdx.x, slice, KS, S, rg, ring_p, xs, pitch, maskall,
                                  spre, bm, dl, rmx, idx_s, jinfo, xo_s, scx, scale, jbase, misc,
                                  xq_bar, abort_flag);
      }
    }
    all_sync();

    if (warp < CW) {
      // ---------------------------------------------------------- compute warps
      const int g = lane >> 2, q = lane & 3;
      const int64_t w0 = k0 / 32;
      const int jb = kRaw ? 0 : jbase[slice];
      int64_t it = 0;
      for (int64_t tile = cta_in_slice; tile < n_tiles; tile += ctas_in_slice, ++it) {
        const int b = static_cast<int>(it & (EW - 1));
        const uint32_t use = static_cast<uint32_t>(it >> 2);
        if (ok) {  // buffer b drained by its epilogue warp (tile it - EW)
          const bool got = mbar_wait(smem_u32(rempty + b), (use & 1u) ^ 1u, abort_flag, a.lim);
          ok = __all_sync(0xffffffffu, got);
        }
        uint8_t* cb_b = cbo + b * (MAXOS * ROWS);
        int c[2][NT][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) c[h][nt][0] = c[h][nt][1] = c[h][nt][2] = c[h][nt][3] = 0;
        for (int st = 0; st < spt; ++st) {
          if (ok) {
            const bool got = mbar_wait(rg.full_bar(), rg.ph, abort_flag, a.lim);
            ok = __all_sync(0xffffffffu, got);
          }
          if (ok) {
            // this warp's 64-byte step of the stage: box warp / 2, chunks cw .. cw + 3 of each
            // (swizzled) 128-byte row; k offset within the slice = stage * CH + 64 * warp.
            // ldmatrix.x4 lane l addresses row l % 8 of matrix l / 8; A matrices are (rows
            // 0-7 | 8-15 of a 16-row group) x (first | second 16 bytes of a 32-byte k step),
            // B matrices the four 16-byte chunks of the step for 8 tokens.
            const uint32_t boxb = ring + rg.s * STAGE_BYTES + (warp >> 1) * (ROWS * BOXW);
            const int cw = (warp & 1) * 4;
            const int mi = lane >> 3, rr = lane & 7;
            uint32_t fa[2][2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int ks = 0; ks < 2; ++ks) {
                const int row = 16 * h + 8 * (mi & 1) + rr;
                const int chunk = cw + 2 * ks + (mi >> 1);
                ldsm_x4(fa[h][ks], boxb + row * BOXW + ((chunk ^ rr) << 4));
              }
            const int64_t kx = static_cast<int64_t>(st) * CH + 64 * warp + 16 * mi;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              uint32_t fb[4];
              ldsm_x4(fb, smem_u32(xs + (nt * 8 + rr) * pitch + kx));
#pragma unroll
              for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                  mma_s8_16816(c[h][nt], fa[h][ks][0], fa[h][ks][1], fa[h][ks][2], fa[h][ks][3],
                               fb[2 * ks], fb[2 * ks + 1]);
            }
            if constexpr (!kRaw) {
              // copy out the bytes of outlier columns in this step: for each one, lane r
              // reads row r's byte from the stage
              const int wl = st * (CH / 32) + 2 * warp;  // slice-local mask word
              const uint32_t mw2[2] = {maskall[w0 + wl], maskall[w0 + wl + 1]};
              if ((mw2[0] | mw2[1]) != 0u) {
#pragma unroll
                for (int hw = 0; hw < 2; ++hw) {
                  const uint32_t mw = mw2[hw];
                  uint32_t bits = mw;
                  while (bits) {
                    const int bp = __ffs(bits) - 1;
                    bits &= bits - 1u;
                    const int jl = spre[wl + hw] + __popc(mw & ((1u << bp) - 1u)) - jb;
                    if (jl < MAXOS && jl + jb < MAXO) {
                      const int col = 32 * hw + bp;  // byte of the warp's 64-byte step
                      const int chunk = cw + (col >> 4);
                      cb_b[jl * ROWS + lane] = lds_u8(boxb + lane * BOXW +
                                                      (((chunk ^ (lane & 7)) << 4) | (col & 15)));
                    }
                  }
                }
              }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(rg.empty_bar());
          }
          rg.advance();
        }
        if (ok) {
          // this warp's 32 x TP partials into buffer b: c[h] covers rows 16h + (g, g + 8),
          // elements 0/1 tokens 2q/2q+1 of row g, 2/3 of row g + 8 (integer adds: the order
          // does not change the sums)
          int32_t* rbuf = red + b * (TP * RP);
#pragma unroll
          for (int h = 0; h < 2; ++h)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
              const int i0 = (nt * 8 + 2 * q) * RP + 16 * h + g;
              atomicAdd(rbuf + i0, c[h][nt][0]);
              atomicAdd(rbuf + i0 + RP, c[h][nt][1]);
              atomicAdd(rbuf + i0 + 8, c[h][nt][2]);
              atomicAdd(rbuf + i0 + RP + 8, c[h][nt][3]);
            }
          __syncwarp();
          if (lane == 0) mbar_arrive(smem_u32(rfull + b));
        }
      }
    } else {
      // ---------------------------------------------------------- epilogue warps
      const int e = warp - EPI0;
      const int rb = static_cast<int>(rec_bytes(T));
      int nos = 0, jb = 0;  // this slice's copied outlier columns: ranks jb .. jb + nos - 1
      if constexpr (!kRaw) {
        jb = jbase[slice];
        nos = jbase[slice + 1] - jb;
        nos = min(nos, min(MAXOS, MAXO - jb));
        if (nos < 0) nos = 0;
      }
      int32_t* rbuf = red + e * (TP * RP);
      const uint8_t* cb_e = cbo + e * (MAXOS * ROWS);
      int64_t it = e;
      for (int64_t tile = cta_in_slice + static_cast<int64_t>(e) * ctas_in_slice; tile < n_tiles;
           tile += static_cast<int64_t>(EW) * ctas_in_slice, it += EW) {
        const uint32_t use = static_cast<uint32_t>(it >> 2);
        const bool got = mbar_wait(smem_u32(rfull + e), use & 1u, abort_flag, a.lim);
        if (!__all_sync(0xffffffffu, got)) break;
        int32_t p[TP];
#pragma unroll
        for (int t = 0; t < TP; ++t) {
          p[t] = rbuf[t * RP + lane];
          rbuf[t * RP + lane] = 0;
        }
        // lane = row of the tile
        uint8_t* rec = a.rec + (tile * S + slice) * rb + lane * 4;
        if constexpr (kRaw) {
#pragma unroll
          for (int t = 0; t < TP; ++t)
            if (t < T) reinterpret_cast<int32_t*>(rec)[t * ROWS] = p[t];
        } else {
          float o[TP];
#pragma unroll
          for (int t = 0; t < TP; ++t) o[t] = 0.0f;
          for (int jl = 0; jl < nos; ++jl) {
            const float cb = static_cast<float>(static_cast<int8_t>(cb_e[jl * ROWS + lane]));
#pragma unroll
            for (int t = 0; t < TP; ++t)
              if (t < T) o[t] = fmaf(__half2float(xo_s[t * MAXO + jb + jl]), cb, o[t]);
          }
#pragma unroll
          for (int t = 0; t < TP; ++t)
            if (t < T)
              reinterpret_cast<float*>(rec)[t * ROWS] =
                  fmaf(static_cast<float>(p[t]), scx[t] * (1.0f / 127.0f), o[t]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(rempty + e));
        fence_acq_rel_gpu();  // the record is visible before the arrival is counted
        __syncwarp();
        int arrivals = 0;
        if (lane == 0) arrivals = tile_arrive(a.cnt + tile, static_cast<uint32_t>(a.epoch));
        arrivals = __shfl_sync(0xffffffffu, arrivals, 0);
        if (arrivals == S) {
          fence_acq_rel_gpu();
          finish_tile<NT, kRaw>(a, tile, S, rb, maskall, idx_s, jinfo, xo_s, misc);
          __syncwarp();
          if (lane == 0)
            *reinterpret_cast<volatile unsigned long long*>(a.cnt + tile) = a.epoch << 32;
        }
      }
    }
  }
  grid_dep_launch();
  __syncthreads();
}

}  // namespace gemv
}  // namespace i8

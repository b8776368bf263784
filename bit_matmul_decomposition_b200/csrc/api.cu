// api.cu -- the C ABI of libi8linear (declared in include/i8linear.h): argument checks,
// workspace layout, TMA descriptors and kernel launches.  One translation unit holds every
// kernel, so the per-device error word is a single module global.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdio>
#include <mutex>
#include <utility>

#include "../../include/i8linear.h"
#include "bwd.cuh"
#include "common.cuh"
#include "gemm.cuh"
#include "gemm_wide.cuh"
#include "gemv.cuh"
#include "quant.cuh"

namespace {

using namespace i8;

constexpr uint64_t kWaitLimitNs = 1000000000ull;  // 1 s for every device-side wait
constexpr int64_t kDecodeMaxT = 16;               // T <= 16 takes the decode kernel
constexpr int64_t kWideMinK = 8192;               // K from which the 256 x 512 GEMM is used
constexpr int kMaxDevices = 64;

// ------------------------------------------------------------------ errors
// The CUDA call behind the last I8_ERR_CUDA returned to this thread (i8_last_error()).
thread_local char g_last_err[192] = "";

void note_cuda(const char* what, int code, const char* name) {
  snprintf(g_last_err, sizeof(g_last_err), "%s failed: %s (%d)", what, name, code);
}

// true when e is cudaSuccess; else records `what` and the error for i8_last_error()
bool cuda_ok(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return true;
  note_cuda(what, static_cast<int>(e), cudaGetErrorName(e));
  return false;
}

// ------------------------------------------------------------------ device info
struct DeviceInfo {
  bool init = false;
  bool sm100 = false;
  int sms = 0;
  bool gemm_attr = false;
  int gemm_clusters = 0;  // co-resident CTA pairs of the GEMM kernel
  int wide_clusters = 0;  // co-resident CTA pairs of the 256 x 512 GEMM kernel
  int bwd_clusters = 0;   // co-resident CTA pairs of the backward fp16 GEMM
  int prep_smem_max = 0;  // dynamic shared memory granted to prepare_kernel
  int smem_optin = 0;     // largest dynamic shared memory a kernel may opt in to
};
std::mutex g_mu;
DeviceInfo g_dev[kMaxDevices];

cudaEvent_t g_prof_start = nullptr;
cudaEvent_t g_prof_stop = nullptr;

size_t p_smem_optin(int dev) {
  int v = 0;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
    return 0;
  return static_cast<size_t>(v);
}

i8_status device_info(DeviceInfo** out) {
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev), "cudaGetDevice")) return I8_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return I8_ERR_UNSUPPORTED;
  // The driver calls of this library (the tensor-map encoder) need the device's context to
  // be current in the calling thread; a thread in which no CUDA runtime has made it current
  // yet (e.g. PyTorch's autograd worker thread) has none: make it current once per thread
  // and device.
  thread_local int ctx_dev = -1;
  if (ctx_dev != dev) {
    if (!cuda_ok(cudaSetDevice(dev), "cudaSetDevice")) return I8_ERR_CUDA;
    ctx_dev = dev;
  }
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.init) {
    cudaDeviceProp p;
    if (!cuda_ok(cudaGetDeviceProperties(&p, dev), "cudaGetDeviceProperties")) return I8_ERR_CUDA;
    d.sm100 = (p.major == 10 && p.minor == 0);
    d.sms = p.multiProcessorCount;
    d.init = true;
  }
  if (!d.sm100) return I8_ERR_UNSUPPORTED;
  if (!d.gemm_attr) {
    const int bytes = static_cast<int>(gemm::SMEM_BYTES);
    const int bwd_bytes = static_cast<int>(bwd::SMEM_BYTES);
    const auto smem_attr = cudaFuncAttributeMaxDynamicSharedMemorySize;
    if (!cuda_ok(cudaFuncSetAttribute(gemm::i8_gemm_tcgen05_kernel<false>, smem_attr, bytes),
                 "cudaFuncSetAttribute(gemm)") ||
        !cuda_ok(cudaFuncSetAttribute(gemm::i8_gemm_tcgen05_kernel<true>, smem_attr, bytes),
                 "cudaFuncSetAttribute(gemm raw)") ||
        !cuda_ok(cudaFuncSetAttribute(gemm::i8_gemm_tcgen05_kernel<false, true>, smem_attr, bytes),
                 "cudaFuncSetAttribute(gemm e4m3)") ||
        !cuda_ok(cudaFuncSetAttribute(bwd::f16_gemm_kernel<false, true>, smem_attr, bwd_bytes),
                 "cudaFuncSetAttribute(f16 gemm)") ||
        !cuda_ok(cudaFuncSetAttribute(gemmw::i8_gemm_wide_kernel<false>, smem_attr,
                                      static_cast<int>(gemmw::SMEM_BYTES)),
                 "cudaFuncSetAttribute(wide gemm)") ||
        !cuda_ok(cudaFuncSetAttribute(gemmw::i8_gemm_wide_kernel<true>, smem_attr,
                                      static_cast<int>(gemmw::SMEM_BYTES)),
                 "cudaFuncSetAttribute(wide gemm e4m3)") ||
        !cuda_ok(cudaFuncSetAttribute(bwd::f16_gemm_kernel<true, true>, smem_attr, bwd_bytes),
                 "cudaFuncSetAttribute(f16 gemm)"))
      return I8_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * d.sms, 1, 1);
    cfg.blockDim = dim3(gemm::THREADS, 1, 1);
    cfg.dynamicSmemBytes = gemm::SMEM_BYTES;
    int clusters = 0;
    if (!cuda_ok(cudaOccupancyMaxActiveClusters(&clusters, gemm::i8_gemm_tcgen05_kernel<false>,
                                                &cfg),
                 "cudaOccupancyMaxActiveClusters(gemm)"))
      return I8_ERR_CUDA;
    if (clusters < 1) return I8_ERR_UNSUPPORTED;
    d.gemm_clusters = clusters;
    cfg.dynamicSmemBytes = bwd::SMEM_BYTES;
    cfg.blockDim = dim3(bwd::THREADS, 1, 1);
    clusters = 0;
    if (!cuda_ok(cudaOccupancyMaxActiveClusters(&clusters, bwd::f16_gemm_kernel<true, true>, &cfg),
                 "cudaOccupancyMaxActiveClusters(f16 gemm)"))
      return I8_ERR_CUDA;
    if (clusters < 1) return I8_ERR_UNSUPPORTED;
    d.bwd_clusters = clusters;
    cfg.dynamicSmemBytes = gemmw::SMEM_BYTES;
    cfg.blockDim = dim3(gemmw::THREADS, 1, 1);
    clusters = 0;
    if (!cuda_ok(cudaOccupancyMaxActiveClusters(&clusters, gemmw::i8_gemm_wide_kernel<false>,
                                                &cfg),
                 "cudaOccupancyMaxActiveClusters(wide gemm)"))
      return I8_ERR_CUDA;
    if (clusters < 1) return I8_ERR_UNSUPPORTED;
    d.wide_clusters = clusters;
    cudaFuncAttributes fa;
    if (!cuda_ok(cudaFuncGetAttributes(&fa, prepare_kernel<false>), "cudaFuncGetAttributes"))
      return I8_ERR_CUDA;
    const int prep_max =
        static_cast<int>(p_smem_optin(dev)) - static_cast<int>(fa.sharedSizeBytes) - 1024;
    if (prep_max < 32 * 1024) return I8_ERR_UNSUPPORTED;
    if (!cuda_ok(cudaFuncSetAttribute(prepare_kernel<false>, smem_attr, prep_max),
                 "cudaFuncSetAttribute(prepare)") ||
        !cuda_ok(cudaFuncSetAttribute(prepare_kernel<true>, smem_attr, prep_max),
                 "cudaFuncSetAttribute(prepare e4m3)"))
      return I8_ERR_CUDA;
    d.prep_smem_max = prep_max;
    d.smem_optin = static_cast<int>(p_smem_optin(dev));
    if (!cuda_ok(cudaFuncSetAttribute(quantize_weight_kernel, smem_attr,
                                      static_cast<int>(kWqRingBytes)),
                 "cudaFuncSetAttribute(quantize_weight)"))
      return I8_ERR_CUDA;
    d.gemm_attr = true;
  }
  *out = &d;
  return I8_OK;
}

// ------------------------------------------------------------------ launches
// Launch with programmatic stream serialization: the kernel may begin while the previous
// kernel on the stream drains, and waits (griddepcontrol.wait) before reading its output.
template <typename... KArgs, typename... Args>
cudaError_t launch_overlapped(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// ------------------------------------------------------------------ checks
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool shape_ok(int64_t T, int64_t K) {
  return T > 0 && K > 0 && (K % 16) == 0 && T <= 0x7fffffffLL && K <= 0x7fffffffLL;
}

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

i8_status launch_status() {
  return cuda_ok(cudaGetLastError(), "kernel launch") ? I8_OK : I8_ERR_CUDA;
}

size_t slice_elems(int64_t rows, int64_t K) {
  return static_cast<size_t>((K + 63) / 64) * static_cast<size_t>(rows) * 64u;
}

// ------------------------------------------------------------------ workspace layout
// Decode batches (T <= 16, K <= 65536) run as one kernel: small T, and each CTA keeps what it
// needs in shared memory.
bool use_decode(int64_t T, int64_t K) { return T <= kDecodeMaxT && K <= gemv::MAX_K; }

struct Workspace {
  size_t mask, idx, n_o, sel, scx, xq, xo, cbo, rec, cnt, gmask, gbm, gbar, total;
  int64_t zero_words;  // words from `mask` on that must be zero when a forward starts
};

// GEMM path: the first region holds the packed outlier mask, the grid-barrier word of the
// fused prepare pass and its outlier-cache update counter; one memset clears them at the
// start of every forward.
// Decode path: the slice records of every 32-row tile, then the control words -- the
// tiles' arrival counters and the words of the cooperative prologue, contiguous from `cnt`
// to the end -- which one memset clears at the start of every decode call.  The words carry
// the launch's epoch in their upper half; a zero upper half never matches an epoch, so no
// bytes left in the workspace by an earlier call of another shape or path, or by another
// user of the memory, can pose as a counter of this launch.
Workspace layout(int64_t T, int64_t N, int64_t K, bool gemm_path = false) {
  Workspace w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  if (!gemm_path && use_decode(T, K)) {
    const size_t n_tiles = static_cast<size_t>((N + gemv::ROWS - 1) / gemv::ROWS);
    w.rec = take(n_tiles * static_cast<size_t>(gemv::num_slices(K)) *
                 static_cast<size_t>(gemv::rec_bytes(T)));
    w.cnt = take(n_tiles * 8);
    w.gmask = take(static_cast<size_t>((K + 31) / 32) * 8);
    w.gbm = take(static_cast<size_t>(T) * static_cast<size_t>((K + gemv::XB - 1) / gemv::XB) * 8);
    w.gbar = take(8);
    w.total = off;
    return w;
  }
  const int64_t words = (K + 31) / 32;
  w.zero_words = words + 2;
  w.mask = take(static_cast<size_t>(w.zero_words) * 4);
  w.idx = take(static_cast<size_t>(K) * 4);
  w.n_o = take(16);
  w.sel = take(16);
  w.scx = take(static_cast<size_t>(T) * 4);
  w.xq = take(static_cast<size_t>(T) * static_cast<size_t>(K));
  w.xo = take(slice_elems(T, K) * 2);
  w.cbo = take(slice_elems(N, K) * 2);
  w.total = off;
  return w;
}

// ------------------------------------------------------------------ outlier cache
// [header: kOcacheHdrWords words + ceil(K/32) mask words, padded to 256 B]
// [CB_o slice: chunk-major [cols / 64][N][64] fp16]
size_t ocache_header_bytes(int64_t K) {
  return align_up(static_cast<size_t>(kOcacheHdrWords + (K + 31) / 32) * 4, 256);
}

// columns a cache of `bytes` holds for an [N, K] weight (0 when it holds none)
int64_t ocache_cols(size_t bytes, int64_t N, int64_t K) {
  const size_t head = ocache_header_bytes(K);
  if (bytes < head) return 0;
  int64_t cols = static_cast<int64_t>((bytes - head) / (static_cast<size_t>(N) * 128u)) * 64;
  const int64_t kmax = (K + 63) / 64 * 64;
  return cols < kmax ? cols : kmax;
}

// ------------------------------------------------------------------ TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// records a failed tensor-map encoding for i8_last_error()
bool encoded(CUresult r) {
  if (r == CUDA_SUCCESS) return true;
  note_cuda("cuTensorMapEncodeTiled", static_cast<int>(r), "CUresult");
  return false;
}

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

// 2-D row-major [outer, inner] tensor, 128-byte-swizzled box [box_outer, box_inner].
bool map_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
            uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    note_cuda("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", 0, "not found");
    return false;
  }
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  return encoded(enc(m, dt, 2, const_cast<void*>(base), dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE));
}

// fp16 output C [rows, cols] for TMA stores of 32 x 32 boxes (cols % 8 == 0).
bool map_c(CUtensorMap* m, void* base, uint64_t cols, uint64_t rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    note_cuda("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", 0, "not found");
    return false;
  }
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t es[2] = {1, 1};
  return encoded(enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, base, dims, strides, box, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE));
}

// Chunk-major outlier slice [chunks][rows][64] fp16; box [1][box_rows][64].
bool map_slice(CUtensorMap* m, const void* base, uint64_t rows, uint64_t chunks,
               uint32_t box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) {
    note_cuda("cudaGetDriverEntryPoint(cuTensorMapEncodeTiled)", 0, "not found");
    return false;
  }
  cuuint64_t dims[3] = {64, rows, chunks};
  cuuint64_t strides[2] = {128, rows * 128};
  cuuint32_t box[3] = {64, box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  return encoded(enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE));
}

// ------------------------------------------------------------------ stage launchers
i8_status run_scan(const void* X, int64_t T, int64_t K, float thr, uint32_t* mask, int32_t* idx,
                   int32_t* n_o, const DeviceInfo& d, cudaStream_t s) {
  const int64_t words = (K + 31) / 32;
  if (!cuda_ok(cudaMemsetAsync(mask, 0, static_cast<size_t>(words) * 4, s), "cudaMemsetAsync"))
    return I8_ERR_CUDA;
  const int64_t groups = K / 8;
  const int64_t gx = (groups + kScanThreads - 1) / kScanThreads;
  const int64_t target = static_cast<int64_t>(d.sms) * 8;
  int64_t gy = (target + gx - 1) / gx;
  if (gy > T) gy = T;
  if (gy < 1) gy = 1;
  const int64_t rows_per_cta = (T + gy - 1) / gy;
  gy = (T + rows_per_cta - 1) / rows_per_cta;
  if (gx > 0x7fffffffLL || gy > 65535) return I8_ERR_INVALID_ARG;
  outlier_scan_kernel<<<dim3(static_cast<unsigned>(gx), static_cast<unsigned>(gy)), kScanThreads,
                        0, s>>>(static_cast<const __half*>(X), T, K, thr, rows_per_cta, mask);
  if (launch_status() != I8_OK) return I8_ERR_CUDA;
  compact_kernel<<<1, kCompactThreads, 0, s>>>(mask, words, idx, n_o);
  return launch_status();
}

i8_status run_quant_rows(const void* A, int64_t R, int64_t K, const uint32_t* mask, int8_t* Q,
                         float* scale, const int32_t* idx, const int32_t* n_o, void* A_o,
                         cudaStream_t s, bool e4m3 = false) {
  quantize_rows_kernel<<<static_cast<unsigned>(R), kQuantThreads, 0, s>>>(
      static_cast<const __half*>(A), R, K, mask, Q, scale, idx, n_o, static_cast<__half*>(A_o),
      e4m3);
  return launch_status();
}

// Step 3 for a whole weight: the streaming quantiser (rows of up to 64 KB), else one CTA
// per row.
i8_status run_quant_weight(const void* W, int64_t N, int64_t K, int8_t* CB, float* SCB,
                           const DeviceInfo& d, cudaStream_t s, bool e4m3 = false) {
  if (K * 2 > kWqMaxRowBytes)
    return run_quant_rows(W, N, K, nullptr, CB, SCB, nullptr, nullptr, nullptr, s, e4m3);
  WqArgs a;
  a.W = static_cast<const __half*>(W);
  a.N = N;
  a.K = K;
  a.CB = CB;
  a.SCB = SCB;
  a.e4m3 = e4m3;
  a.R = wq_rows_per_stage(K);
  a.stages = (N + a.R - 1) / a.R;
  a.slots = wq_slots(K);
  a.wait_limit_ns = kWaitLimitNs;
  const int64_t grid = a.stages < 2 * d.sms ? a.stages : 2 * d.sms;   // two CTAs per SM
  const size_t smem = static_cast<size_t>(a.slots) * static_cast<size_t>(a.R * K * 2);
  quantize_weight_kernel<<<static_cast<unsigned>(grid), kWqThreads, smem, s>>>(a);
  return launch_status();
}

// Fused steps 1 + 2 (+ the fp16 outlier slices): one cooperative launch.
// mask must hold ceil(K/32) + 1 words; the last one is the grid-barrier counter.
// `zero_words` words from `mask` on are cleared first (at least the mask and the barrier
// word, ceil(K/32) + 1).
// With an outlier cache (`ocache` non-NULL, `ocache_cols` columns), CB_o is kept there
// across calls and *cbo_sel tells the GEMM which slice holds this call's CB_o.
i8_status run_prepare(const void* X, int64_t T, int64_t K, float thr, uint32_t* mask,
                      int64_t zero_words, int32_t* idx, int32_t* n_o, int8_t* Xq, float* SCx,
                      void* X_o, const int8_t* CB, int64_t N, void* CB_o, const DeviceInfo& d,
                      cudaStream_t s, uint8_t* ocache = nullptr, int64_t ocols = 0,
                      int32_t* cbo_sel = nullptr, bool e4m3 = false) {
  if (!cuda_ok(cudaMemsetAsync(mask, 0, static_cast<size_t>(zero_words) * 4, s), "cudaMemsetAsync"))
    return I8_ERR_CUDA;
  const int64_t G0 = d.sms;
  const int64_t rows_per_cta = (T + G0 - 1) / G0;
  const size_t head = prepare_smem_bytes(K, 0, rows_per_cta);
  const size_t budget = static_cast<size_t>(d.prep_smem_max);
  if (head + 16 > budget) return I8_ERR_INVALID_ARG;
  int64_t cache_rows = static_cast<int64_t>((budget - head) / prepare_row_bytes(K));
  if (cache_rows > rows_per_cta) cache_rows = rows_per_cta;
  if (cache_rows * K * 2 > static_cast<int64_t>(kPrepChunk) * kPrepMaxChunks)
    cache_rows = static_cast<int64_t>(kPrepChunk) * kPrepMaxChunks / (K * 2);
  const size_t smem = prepare_smem_bytes(K, cache_rows, rows_per_cta);
  int per_sm = 0;
  const void* kernel = e4m3 ? reinterpret_cast<const void*>(prepare_kernel<true>)
                            : reinterpret_cast<const void*>(prepare_kernel<false>);
  if (!cuda_ok(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kPrepThreads,
                                                             smem),
               "cudaOccupancyMaxActiveBlocksPerMultiprocessor(prepare)"))
    return I8_ERR_CUDA;
  if (per_sm < 1) return I8_ERR_INVALID_ARG;
  const int grid = d.sms;  // one CTA per SM: every CTA is resident for the grid barrier
  PrepArgs a;
  a.X = static_cast<const __half*>(X);
  a.T = T;
  a.K = K;
  a.thr = thr;
  a.mask = mask;
  a.idx_out = idx;
  a.n_o_out = n_o;
  a.Xq = Xq;
  a.SCx = SCx;
  a.X_o = static_cast<__half*>(X_o);
  a.CB = CB;
  a.N = N;
  a.CB_o = static_cast<__half*>(CB_o);
  a.ocache = reinterpret_cast<uint32_t*>(ocache);
  a.ocache_CB_o =
      ocache ? reinterpret_cast<__half*>(ocache + ocache_header_bytes(K)) : nullptr;
  a.ocache_cols = ocache ? ocols : 0;
  a.cbo_sel = cbo_sel;
  a.rows_per_cta = rows_per_cta;
  a.cache_rows = cache_rows;
  a.cache_bytes_all = cache_rows * K * 2;
  a.wait_limit_ns = kWaitLimitNs;
  void* params[] = {&a};
  if (!cuda_ok(cudaLaunchCooperativeKernel(kernel, dim3(grid),
                                  dim3(kPrepThreads), params, smem, s), "cudaLaunchCooperativeKernel"))
    return I8_ERR_CUDA;
  return launch_status();
}

// tcgen05 GEMM (pairs of CTAs, 256 x 256 tiles); raw=true writes the int32 accumulator.
// B_c (ocols columns) is the outlier cache's CB_o slice, read instead of B_o when the
// device word *cbo_sel is nonzero.
// Long K-loops with enough tiles to fill the GPU several times take the 256 x 512 tiles
// (a quarter less operand feed per multiply-add; the epilogue is not overlapped, which a
// long K-loop hides).
bool use_wide(int64_t T, int64_t N, int64_t K, const DeviceInfo& d) {
  const int64_t m_tiles = (T + gemm::TM - 1) / gemm::TM;
  const int64_t wide_tiles = m_tiles * ((N + gemmw::TN - 1) / gemmw::TN);
  return K >= kWideMinK && wide_tiles >= 4 * static_cast<int64_t>(d.wide_clusters);
}

i8_status run_gemm(bool raw, const int8_t* A, int64_t T, int64_t K, const int8_t* B, int64_t N,
                   const void* A_o, const void* B_o, const int32_t* n_o, const float* SCx,
                   const float* SCB, const void* bias, void* C, int32_t* acc,
                   const DeviceInfo& d, cudaStream_t s, const void* B_c = nullptr,
                   int64_t ocols = 0, const int32_t* cbo_sel = nullptr, bool e4m3 = false) {
  CUtensorMap tA, tB, tAo, tBo, tBc, tC;
  if (!map_2d(&tA, CU_TENSOR_MAP_DATA_TYPE_UINT8, A, K, T, K, gemm::BK, gemm::HM) ||
      !map_2d(&tB, CU_TENSOR_MAP_DATA_TYPE_UINT8, B, K, N, K, gemm::BK, gemm::HN))
    return I8_ERR_CUDA;
  if (raw) {
    tAo = tA;
    tBo = tB;
  } else {
    const uint64_t chunks = static_cast<uint64_t>((K + 63) / 64);
    if (!map_slice(&tAo, A_o, T, chunks, gemm::HM) || !map_slice(&tBo, B_o, N, chunks, gemm::HN))
      return I8_ERR_CUDA;
  }
  tBc = tBo;
  // C goes out by TMA stores when its row pitch allows a tensor map (N % 8 == 0)
  tC = tA;
  const bool c_tma = !raw && C != nullptr && (N % 8) == 0;
  if (c_tma && !map_c(&tC, C, static_cast<uint64_t>(N), static_cast<uint64_t>(T)))
    return I8_ERR_CUDA;
  if (!raw && B_c != nullptr && cbo_sel != nullptr &&
      !map_slice(&tBc, B_c, N, static_cast<uint64_t>(ocols / 64), gemm::HN))
    return I8_ERR_CUDA;
  gemm::Args a;
  a.T = static_cast<int>(T);
  a.N = static_cast<int>(N);
  a.K = static_cast<int>(K);
  a.m_tiles = static_cast<int>((T + gemm::TM - 1) / gemm::TM);
  a.n_tiles = static_cast<int>((N + gemm::TN - 1) / gemm::TN);
  a.k_blocks = static_cast<int>((K + gemm::BK - 1) / gemm::BK);
  a.n_outliers = raw ? nullptr : n_o;
  a.cbo_sel = (raw || B_c == nullptr) ? nullptr : cbo_sel;
  a.SCx = SCx;
  a.SCB = SCB;
  a.bias = static_cast<const __half*>(bias);
  a.C = static_cast<__half*>(C);
  a.acc_out = acc;
  a.c_tma = c_tma;
  a.wait_limit_ns = kWaitLimitNs;
  const int64_t wide_tiles = static_cast<int64_t>(a.m_tiles) * ((N + gemmw::TN - 1) / gemmw::TN);
  if (!raw && use_wide(T, N, K, d)) {
    a.n_tiles = static_cast<int>((N + gemmw::TN - 1) / gemmw::TN);
    const int wc = static_cast<int>(wide_tiles < d.wide_clusters ? wide_tiles : d.wide_clusters);
    const cudaError_t e =
        e4m3 ? launch_overlapped(gemmw::i8_gemm_wide_kernel<true>, dim3(2 * wc),
                                 dim3(gemmw::THREADS), gemmw::SMEM_BYTES, s, tA, tB, tAo, tBo,
                                 tBc, tC, a)
             : launch_overlapped(gemmw::i8_gemm_wide_kernel<false>, dim3(2 * wc),
                                 dim3(gemmw::THREADS), gemmw::SMEM_BYTES, s, tA, tB, tAo, tBo,
                                 tBc, tC, a);
    return cuda_ok(e, "kernel launch") ? launch_status() : I8_ERR_CUDA;
  }
  const int64_t tiles = static_cast<int64_t>(a.m_tiles) * a.n_tiles;
  const int clusters = static_cast<int>(tiles < d.gemm_clusters ? tiles : d.gemm_clusters);
  cudaError_t e;
  if (e4m3 && !raw)
    e = launch_overlapped(gemm::i8_gemm_tcgen05_kernel<false, true>, dim3(2 * clusters),
                          dim3(gemm::THREADS), gemm::SMEM_BYTES, s, tA, tB, tAo, tBo, tBc, tC, a);
  else if (raw)
    e = launch_overlapped(gemm::i8_gemm_tcgen05_kernel<true>, dim3(2 * clusters),
                          dim3(gemm::THREADS), gemm::SMEM_BYTES, s, tA, tB, tAo, tBo, tBc, tC, a);
  else
    e = launch_overlapped(gemm::i8_gemm_tcgen05_kernel<false>, dim3(2 * clusters),
                          dim3(gemm::THREADS), gemm::SMEM_BYTES, s, tA, tB, tAo, tBo, tBc, tC, a);
  return cuda_ok(e, "kernel launch") ? launch_status() : I8_ERR_CUDA;
}

// Backward fp16 GEMM: C[M, Nc] = sum_r A(m, r) B(n, r); a_mn / b_mn: the operand's rows run
// along m / n (MN-major) instead of the reduction.  lda / ldb: elements per row in memory.
i8_status run_f16_gemm(bool a_mn, const void* A, int64_t lda, bool b_mn, const void* B,
                       int64_t ldb, int64_t M, int64_t Nc, int64_t R, void* C,
                       const DeviceInfo& d, cudaStream_t s) {
  CUtensorMap tA, tB, tC;
  const auto F16 = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
  // K-major: [M rows][R] with 128 x 64 boxes; MN-major: [R rows][M] with 64 x 64 boxes
  const bool okA = a_mn ? map_2d(&tA, F16, A, M, R, lda * 2, 64, 64)
                        : map_2d(&tA, F16, A, R, M, lda * 2, 64, 128);
  const bool okB = b_mn ? map_2d(&tB, F16, B, Nc, R, ldb * 2, 64, 64)
                        : map_2d(&tB, F16, B, R, Nc, ldb * 2, 64, 128);
  if (!okA || !okB) return I8_ERR_CUDA;
  tC = tA;
  const bool c_tma = (Nc % 8) == 0;
  if (c_tma && !map_c(&tC, C, static_cast<uint64_t>(Nc), static_cast<uint64_t>(M)))
    return I8_ERR_CUDA;
  bwd::Args a;
  a.M = static_cast<int>(M);
  a.Nc = static_cast<int>(Nc);
  a.R = static_cast<int>(R);
  a.m_tiles = static_cast<int>((M + bwd::TM - 1) / bwd::TM);
  a.n_tiles = static_cast<int>((Nc + bwd::TN - 1) / bwd::TN);
  a.k_blocks = static_cast<int>((R + bwd::BK - 1) / bwd::BK);
  a.C = static_cast<__half*>(C);
  a.ldc = static_cast<int>(Nc);
  a.c_tma = c_tma;
  a.wait_limit_ns = kWaitLimitNs;
  const int64_t tiles = static_cast<int64_t>(a.m_tiles) * a.n_tiles;
  const int clusters = static_cast<int>(tiles < d.bwd_clusters ? tiles : d.bwd_clusters);
  cudaError_t e;
  if (a_mn && b_mn)
    e = launch_overlapped(bwd::f16_gemm_kernel<true, true>, dim3(2 * clusters),
                          dim3(bwd::THREADS), bwd::SMEM_BYTES, s, tA, tB, tC, a);
  else if (!a_mn && b_mn)
    e = launch_overlapped(bwd::f16_gemm_kernel<false, true>, dim3(2 * clusters),
                          dim3(bwd::THREADS), bwd::SMEM_BYTES, s, tA, tB, tC, a);
  else
    return I8_ERR_INVALID_ARG;
  return cuda_ok(e, "kernel launch") ? launch_status() : I8_ERR_CUDA;
}

// decode: one launch of the decode kernel (forward from X, or the raw product of codes)
std::atomic<unsigned long long> g_epoch{0};

// The prologue of the forward reads all of X in every CTA when X fits eight ring stages
// (128 KB, ~1 us per stage); beyond that the CTAs split the scan and meet at one grid
// barrier (cooperative launch).
bool decode_coop(bool raw, int64_t T, int64_t K) {
  return !raw && T * K * 2 > 8 * static_cast<int64_t>(gemv::STAGE_BYTES);
}

i8_status run_decode(bool raw, const void* X, const int8_t* Xq, int64_t T, int64_t K,
                     const int8_t* CB, int64_t N, float thr, const float* SCB, const void* bias,
                     void* C, int32_t* acc, uint8_t* ws, const Workspace& w,
                     const DeviceInfo& d, cudaStream_t s) {
  const int nt = T <= 8 ? 1 : 2;
  const size_t smem = gemv::smem_bytes(nt, K);
  if (smem > static_cast<size_t>(d.smem_optin)) return I8_ERR_INVALID_ARG;
  CUtensorMap tCB;
  if (!map_2d(&tCB, CU_TENSOR_MAP_DATA_TYPE_UINT8, CB, K, N, K, gemv::BOXW, gemv::ROWS))
    return I8_ERR_CUDA;
  // the tile counters and the prologue's words (contiguous from cnt) start at zero
  if (!cuda_ok(cudaMemsetAsync(ws + w.cnt, 0, w.total - w.cnt, s), "cudaMemsetAsync")) return I8_ERR_CUDA;
  const int S = static_cast<int>(gemv::num_slices(K));
  int grid = (d.sms / S) * S;  // one CTA per SM, the same number of CTAs on every slice
  if (grid > 255) grid = (255 / S) * S;  // arrival counts are 8-bit
  if (grid < S) grid = S;
  gemv::Args a;
  a.X = static_cast<const __half*>(X);
  a.Xq = Xq;
  a.T = static_cast<int>(T);
  a.N = N;
  a.K = K;
  a.thr = thr;
  a.CB = CB;
  a.SCB = SCB;
  a.bias = static_cast<const __half*>(bias);
  a.C = static_cast<__half*>(C);
  a.acc = acc;
  a.rec = ws + w.rec;
  a.cnt = reinterpret_cast<unsigned long long*>(ws + w.cnt);
  a.epoch = g_epoch.fetch_add(1) % 0xffffffffull + 1;  // 1 .. 2^32 - 1
  a.lim = kWaitLimitNs;
  a.coop = decode_coop(raw, T, K);
  a.gmask = reinterpret_cast<unsigned long long*>(ws + w.gmask);
  a.gbm = reinterpret_cast<unsigned long long*>(ws + w.gbm);
  a.gbar = reinterpret_cast<unsigned long long*>(ws + w.gbar);
  auto go = [&](auto kernel) -> cudaError_t {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    if (!a.coop)
      return launch_overlapped(kernel, dim3(static_cast<unsigned>(grid)), dim3(gemv::THREADS),
                               smem, s, tCB, a);
    // every CTA must be resident for the grid barriers
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(gemv::THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute at[2];
    at[0].id = cudaLaunchAttributeCooperative;
    at[0].val.cooperative = 1;
    at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, tCB, a);
  };
  cudaError_t e;
  if (nt == 1)
    e = raw ? go(gemv::decode_kernel<1, true>) : go(gemv::decode_kernel<1, false>);
  else
    e = raw ? go(gemv::decode_kernel<2, true>) : go(gemv::decode_kernel<2, false>);
  return cuda_ok(e, "kernel launch") ? launch_status() : I8_ERR_CUDA;
}

__global__ void bounded_wait_selftest_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the wait must give up after limit_ns and flag it
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0u, &abort_flag, limit_ns);
}

// ------------------------------------------------------------------ fixed scratch
// Scratch for i8_linear_forward_noalloc: a file-scope device array, so that entry point
// needs no allocation.  Every GPU that loads this library holds these bytes until the
// process exits.  In host code the symbol is only a stand-in for the array; its device
// address comes from cudaGetSymbolAddress, once per device, on that device.
constexpr size_t kStaticScratchBytes = size_t(32) << 20;  // 32 MiB
__device__ __align__(256) uint8_t g_static_scratch[kStaticScratchBytes];

void* g_static_scratch_addr[kMaxDevices] = {};

// Device address of g_static_scratch on the current device (looked up on first use).
i8_status static_scratch_address(void** out) {
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev), "cudaGetDevice")) return I8_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return I8_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_static_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (!cuda_ok(cudaGetSymbolAddress(&p, g_static_scratch), "cudaGetSymbolAddress") ||
        p == nullptr)
      return I8_ERR_CUDA;
    g_static_scratch_addr[dev] = p;
  }
  *out = g_static_scratch_addr[dev];
  return I8_OK;
}

// The forward of every entry point: int8 codes (with `cache`, ocols columns, or without:
// NULL), or e4m3 codes (no cache; the prepare pass and the GEMM for every T).
i8_status forward_impl(const void* X, int64_t T, int64_t K, const int8_t* CB, const float* SCB,
                       const void* bias, int64_t N, float threshold, void* C, void* workspace,
                       size_t workspace_bytes, uint8_t* cache, int64_t ocols, void* stream,
                       bool e4m3 = false) {
  if (!X || !CB || !SCB || !C || !workspace) return I8_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(CB) || !aligned16(SCB) || !aligned16(C) ||
      !aligned16(workspace) || (bias && !aligned16(bias)))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL || threshold != threshold)
    return I8_ERR_INVALID_ARG;
  const Workspace w = layout(T, N, K, e4m3);
  if (workspace_bytes < w.total) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const bool prof = g_prof_start != nullptr && g_prof_stop != nullptr;
  if (!e4m3 && use_decode(T, K)) {
    // (the decode kernel takes the outlier columns' codes out of its own CB stream)
    if (prof && !cuda_ok(cudaEventRecord(g_prof_start, s), "cudaEventRecord")) return I8_ERR_CUDA;
    st = run_decode(false, X, nullptr, T, K, CB, N, threshold, SCB, bias, C, nullptr, ws, w, *d,
                    s);
    if (st != I8_OK) return st;
    if (prof && !cuda_ok(cudaEventRecord(g_prof_stop, s), "cudaEventRecord")) return I8_ERR_CUDA;
    return I8_OK;
  }
  uint32_t* mask = reinterpret_cast<uint32_t*>(ws + w.mask);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + w.idx);
  int32_t* n_o = reinterpret_cast<int32_t*>(ws + w.n_o);
  int32_t* sel = cache ? reinterpret_cast<int32_t*>(ws + w.sel) : nullptr;
  float* SCx = reinterpret_cast<float*>(ws + w.scx);
  int8_t* Xq = reinterpret_cast<int8_t*>(ws + w.xq);
  void* X_o = ws + w.xo;
  void* CB_o = ws + w.cbo;
  st = run_prepare(X, T, K, threshold, mask, w.zero_words, idx, n_o, Xq, SCx, X_o, CB, N, CB_o,
                   *d, s, cache, ocols, sel, e4m3);
  if (st != I8_OK) return st;
  if (prof && !cuda_ok(cudaEventRecord(g_prof_start, s), "cudaEventRecord")) return I8_ERR_CUDA;
  st = run_gemm(false, Xq, T, K, CB, N, X_o, CB_o, n_o, SCx, SCB, bias, C, nullptr, *d, s,
                cache ? cache + ocache_header_bytes(K) : nullptr, ocols, sel, e4m3);
  if (st != I8_OK) return st;
  if (prof && !cuda_ok(cudaEventRecord(g_prof_stop, s), "cudaEventRecord")) return I8_ERR_CUDA;
  return I8_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

const char* i8_last_error(void) { return g_last_err; }

const char* i8_status_string(i8_status s) {
  switch (s) {
    case I8_OK: return "I8_OK";
    case I8_ERR_INVALID_ARG: return "I8_ERR_INVALID_ARG";
    case I8_ERR_UNSUPPORTED: return "I8_ERR_UNSUPPORTED";
    case I8_ERR_CUDA: return "I8_ERR_CUDA";
    case I8_ERR_TIMEOUT: return "I8_ERR_TIMEOUT";
    case I8_ERR_DEVICE: return "I8_ERR_DEVICE";
  }
  return "I8_UNKNOWN_STATUS";
}

size_t i8_outlier_slice_elems(int64_t rows, int64_t K) {
  if (rows <= 0 || K <= 0) return 0;
  return slice_elems(rows, K);
}

size_t i8_linear_workspace_size(int64_t T, int64_t N, int64_t K) {
  if (!shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL) return 0;
  return layout(T, N, K).total;
}

i8_status i8_forward_kernel(int64_t T, int64_t N, int64_t K, int32_t* kind) {
  if (!kind || !shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL) return I8_ERR_INVALID_ARG;
  if (use_decode(T, K)) {
    *kind = I8_KERNEL_DECODE;
    return I8_OK;
  }
  DeviceInfo* d;
  const i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  *kind = use_wide(T, N, K, *d) ? I8_KERNEL_GEMM_WIDE : I8_KERNEL_GEMM;
  return I8_OK;
}

i8_status i8_quantize_weight(const void* W, int64_t N, int64_t K, int8_t* CB, float* SCB,
                             void* stream) {
  if (!W || !CB || !SCB || !aligned16(W) || !aligned16(CB) || !aligned16(SCB)) return I8_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  return run_quant_weight(W, N, K, CB, SCB, *d, static_cast<cudaStream_t>(stream));
}

i8_status i8_outlier_scan(const void* X, int64_t T, int64_t K, float threshold, uint32_t* col_mask,
                          int32_t* outlier_idx, int32_t* n_outliers, void* stream) {
  if (!X || !col_mask || !outlier_idx || !n_outliers || !aligned16(X) || !aligned16(col_mask) ||
      !aligned16(outlier_idx) || !aligned16(n_outliers))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || threshold != threshold) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  return run_scan(X, T, K, threshold, col_mask, outlier_idx, n_outliers, *d,
                  static_cast<cudaStream_t>(stream));
}

i8_status i8_quantize_act(const void* X, int64_t T, int64_t K, const uint32_t* col_mask,
                          const int32_t* outlier_idx, const int32_t* n_outliers, int8_t* Xq,
                          float* SCx, void* X_o, void* stream) {
  if (!X || !col_mask || !outlier_idx || !n_outliers || !Xq || !SCx || !X_o)
    return I8_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(col_mask) || !aligned16(outlier_idx) || !aligned16(Xq) ||
      !aligned16(SCx) || !aligned16(X_o) || !aligned16(n_outliers))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K)) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  return run_quant_rows(X, T, K, col_mask, Xq, SCx, outlier_idx, n_outliers, X_o,
                        static_cast<cudaStream_t>(stream));
}

i8_status i8_prepare_act(const void* X, int64_t T, int64_t K, float threshold,
                         uint32_t* col_mask, int32_t* outlier_idx, int32_t* n_outliers,
                         int8_t* Xq, float* SCx, void* X_o, void* stream) {
  if (!X || !col_mask || !outlier_idx || !n_outliers || !Xq || !SCx || !X_o)
    return I8_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(col_mask) || !aligned16(outlier_idx) || !aligned16(Xq) ||
      !aligned16(SCx) || !aligned16(X_o) || !aligned16(n_outliers))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || threshold != threshold) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  return run_prepare(X, T, K, threshold, col_mask, (K + 31) / 32 + 1, outlier_idx, n_outliers,
                     Xq, SCx, X_o, nullptr, 0, nullptr, *d, static_cast<cudaStream_t>(stream));
}

i8_status i8_linear_forward(const void* X, int64_t T, int64_t K, const int8_t* CB,
                            const float* SCB, const void* bias, int64_t N, float threshold,
                            void* C, void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(X, T, K, CB, SCB, bias, N, threshold, C, workspace, workspace_bytes,
                      nullptr, 0, stream);
}

size_t i8_outlier_cache_size(int64_t N, int64_t K, int64_t max_cols) {
  if (N <= 0 || N > 0x7fffffffLL || !shape_ok(1, K) || max_cols <= 0) return 0;
  const int64_t kmax = (K + 63) / 64 * 64;
  const int64_t cols = max_cols < kmax ? (max_cols + 63) / 64 * 64 : kmax;
  return ocache_header_bytes(K) + slice_elems(N, cols) * 2;
}

i8_status i8_outlier_cache_reset(void* cache, size_t cache_bytes, void* stream) {
  if (!cache || !aligned16(cache) || cache_bytes < kOcacheHdrWords * 4) return I8_ERR_INVALID_ARG;
  if (cudaMemsetAsync(cache, 0, kOcacheHdrWords * 4, static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return I8_ERR_CUDA;
  return I8_OK;
}

size_t i8_linear_workspace_size_e4m3(int64_t T, int64_t N, int64_t K) {
  if (!shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL) return 0;
  return layout(T, N, K, true).total;
}

i8_status i8_quantize_weight_e4m3(const void* W, int64_t N, int64_t K, uint8_t* CB, float* SCB,
                                  void* stream) {
  if (!W || !CB || !SCB || !aligned16(W) || !aligned16(CB) || !aligned16(SCB)) return I8_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  return run_quant_weight(W, N, K, reinterpret_cast<int8_t*>(CB), SCB, *d,
                          static_cast<cudaStream_t>(stream), true);
}

i8_status i8_prepare_act_e4m3(const void* X, int64_t T, int64_t K, float threshold,
                              uint32_t* col_mask, int32_t* outlier_idx, int32_t* n_outliers,
                              uint8_t* Xq, float* SCx, void* X_o, void* stream) {
  if (!X || !col_mask || !outlier_idx || !n_outliers || !Xq || !SCx || !X_o)
    return I8_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(col_mask) || !aligned16(outlier_idx) || !aligned16(Xq) ||
      !aligned16(SCx) || !aligned16(X_o) || !aligned16(n_outliers))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || threshold != threshold) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  return run_prepare(X, T, K, threshold, col_mask, (K + 31) / 32 + 1, outlier_idx, n_outliers,
                     reinterpret_cast<int8_t*>(Xq), SCx, X_o, nullptr, 0, nullptr, *d,
                     static_cast<cudaStream_t>(stream), nullptr, 0, nullptr, true);
}

i8_status i8_linear_forward_e4m3(const void* X, int64_t T, int64_t K, const uint8_t* CB,
                                 const float* SCB, const void* bias, int64_t N, float threshold,
                                 void* C, void* workspace, size_t workspace_bytes, void* stream) {
  return forward_impl(X, T, K, reinterpret_cast<const int8_t*>(CB), SCB, bias, N, threshold, C,
                      workspace, workspace_bytes, nullptr, 0, stream, true);
}

i8_status i8_linear_forward_cached(const void* X, int64_t T, int64_t K, const int8_t* CB,
                                   const float* SCB, const void* bias, int64_t N,
                                   float threshold, void* C, void* workspace,
                                   size_t workspace_bytes, void* cache, size_t cache_bytes,
                                   void* stream) {
  if (!cache || !aligned16(cache)) return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL) return I8_ERR_INVALID_ARG;
  const int64_t ocols = ocache_cols(cache_bytes, N, K);
  if (ocols < 64) return I8_ERR_INVALID_ARG;
  return forward_impl(X, T, K, CB, SCB, bias, N, threshold, C, workspace, workspace_bytes,
                      static_cast<uint8_t*>(cache), ocols, stream);
}

i8_status i8_igemm_s32(const int8_t* A, int64_t T, int64_t K, const int8_t* B, int64_t N,
                       int32_t* acc, void* workspace, size_t workspace_bytes, void* stream) {
  if (!A || !B || !acc || !workspace || !aligned16(A) || !aligned16(B) || !aligned16(acc) ||
      !aligned16(workspace))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL || K > 133144) return I8_ERR_INVALID_ARG;
  const Workspace w = layout(T, N, K);
  if (workspace_bytes < w.total) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!use_decode(T, K))
    return run_gemm(true, A, T, K, B, N, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr,
                    nullptr, acc, *d, s);
  return run_decode(true, nullptr, A, T, K, B, N, 0.0f, nullptr, nullptr, nullptr, acc,
                    static_cast<uint8_t*>(workspace), w, *d, s);
}

i8_status i8_linear_backward_input(const void* dY, int64_t T, int64_t N, const void* W,
                                   int64_t K, void* dX, void* stream) {
  if (!dY || !W || !dX || !aligned16(dY) || !aligned16(W) || !aligned16(dX))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL || (N % 8) != 0) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  return run_f16_gemm(false, dY, N, true, W, K, T, K, N, dX, *d,
                      static_cast<cudaStream_t>(stream));
}

i8_status i8_linear_backward_weight(const void* dY, const void* X, int64_t T, int64_t N,
                                    int64_t K, void* dW, void* stream) {
  if (!dY || !X || !dW || !aligned16(dY) || !aligned16(X) || !aligned16(dW))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL || (N % 8) != 0) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  return run_f16_gemm(true, dY, N, true, X, K, N, K, T, dW, *d,
                      static_cast<cudaStream_t>(stream));
}

i8_status i8_bias_grad(const void* dY, int64_t T, int64_t N, void* db, void* stream) {
  if (!dY || !db || !aligned16(dY) || !aligned16(db)) return I8_ERR_INVALID_ARG;
  if (T <= 0 || T > 0x7fffffffLL || N <= 0 || N > 0x7fffffffLL || (N % 8) != 0)
    return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  bwd::bias_grad_kernel<<<static_cast<unsigned>((N + 63) / 64), bwd::kBiasThreads, 0,
                          static_cast<cudaStream_t>(stream)>>>(
      static_cast<const __half*>(dY), T, N, static_cast<__half*>(db));
  return launch_status();
}

static i8_status dequantize(const void* CB, const float* SCB, int64_t N, int64_t K, void* W,
                            void* stream, bool e4m3) {
  if (!CB || !SCB || !W || !aligned16(CB) || !aligned16(SCB) || !aligned16(W))
    return I8_ERR_INVALID_ARG;
  if (!shape_ok(N, K)) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  const int64_t groups = N * K / 16;
  int64_t grid = (groups + bwd::kDequantThreads - 1) / bwd::kDequantThreads;
  if (grid > static_cast<int64_t>(d->sms) * 16) grid = static_cast<int64_t>(d->sms) * 16;
  bwd::dequantize_kernel<<<static_cast<unsigned>(grid), bwd::kDequantThreads, 0,
                           static_cast<cudaStream_t>(stream)>>>(
      static_cast<const int8_t*>(CB), SCB, N, K, static_cast<__half*>(W), e4m3);
  return launch_status();
}

i8_status i8_dequantize_weight(const int8_t* CB, const float* SCB, int64_t N, int64_t K, void* W,
                               void* stream) {
  return dequantize(CB, SCB, N, K, W, stream, false);
}

i8_status i8_dequantize_weight_e4m3(const uint8_t* CB, const float* SCB, int64_t N, int64_t K,
                                    void* W, void* stream) {
  return dequantize(CB, SCB, N, K, W, stream, true);
}

i8_status i8_sync_status(void* stream) {
  if (!cuda_ok(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)), "cudaStreamSynchronize")) return I8_ERR_CUDA;
  unsigned int word = 0;
  if (!cuda_ok(cudaMemcpyFromSymbol(&word, i8::g_error_word, sizeof(word)), "cudaMemcpyFromSymbol"))
    return I8_ERR_CUDA;
  if (word == 0) return I8_OK;
  const unsigned int zero = 0;
  if (!cuda_ok(cudaMemcpyToSymbol(i8::g_error_word, &zero, sizeof(zero)), "cudaMemcpyToSymbol")) return I8_ERR_CUDA;
  if (word & i8::kErrWaitTimeout) return I8_ERR_TIMEOUT;
  return I8_ERR_DEVICE;
}

i8_status i8_set_profile_events(void* start_event, void* stop_event) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_prof_start = static_cast<cudaEvent_t>(start_event);
  g_prof_stop = static_cast<cudaEvent_t>(stop_event);
  return I8_OK;
}

i8_status i8_selftest_bounded_wait(int64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  bounded_wait_selftest_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint64_t>(limit_ns));
  return launch_status();
}

i8_status i8_linear_forward_noalloc(const void* X, int64_t T, int64_t K, const int8_t* CB,
                                    const float* SCB, const void* bias, int64_t N,
                                    float threshold, void* C, void* stream) {
  if (!X || !CB || !SCB || !C) return I8_ERR_INVALID_ARG;
  if (!shape_ok(T, K) || N <= 0 || N > 0x7fffffffLL) return I8_ERR_INVALID_ARG;
  if (layout(T, N, K).total > kStaticScratchBytes) return I8_ERR_INVALID_ARG;
  DeviceInfo* d;
  i8_status st = device_info(&d);
  if (st != I8_OK) return st;
  void* scratch = nullptr;
  st = static_scratch_address(&scratch);
  if (st != I8_OK) return st;
  return i8_linear_forward(X, T, K, CB, SCB, bias, N, threshold, C, scratch,
                           kStaticScratchBytes, stream);
}


}  // extern "C"

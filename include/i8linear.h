/*
 * i8linear.h -- C ABI of libi8linear: the LLM.int8() mixed-precision decomposed linear
 * layer on NVIDIA B200 (sm_100a).
 *
 * The layer, as the pages describe it ("A Gentle Introduction to 8-bit Matrix
 * Multiplication for transformers at scale", Hugging Face blog; sections
 * "LLM.int8() 的总结" and "内部的 MatMul"):
 *   1. find the outlier feature columns of the fp16 hidden states X (magnitude >= 6);
 *   2. quantise the remaining columns of X row-wise (one absmax per token);
 *   3. quantise the weight W once per output channel into int8 codes CB and scales SCB;
 *   4. multiply the int8 parts with an int32 accumulator;
 *   5. dequantise by the outer product of the two absmax vectors;
 *   6. multiply the outlier columns in fp16 against the recovered weights CB*SCB/127,
 *      add both parts and the bias, and return fp16.
 *
 * Conventions for every call
 *   - fp16 means IEEE 754 binary16; it is passed as `const void*` / `void*`.
 *   - All tensors are dense and row-major.  X is [T, K] (T tokens, K input features);
 *     W and CB are [N, K] (the nn.Linear [out, in] layout); C is [T, N].
 *   - Every pointer is a DEVICE pointer, owned and allocated by the caller (for example
 *     by PyTorch), 16-byte aligned.  No call allocates device memory; the only device
 *     memory the library holds is the fixed scratch array of i8_linear_forward_noalloc.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls only enqueue
 *     work; they return before the GPU finishes and never synchronise, except
 *     i8_sync_status().
 *   - Arguments are validated on the host before anything is launched; a violation
 *     returns I8_ERR_INVALID_ARG and enqueues nothing.  Shapes: T, N, K > 0 and
 *     K % 16 == 0 (the int8 row pitch must be a multiple of 16 bytes for TMA).
 *   - The calls need an sm_100 device (B200); another device gives I8_ERR_UNSUPPORTED.
 *   - Every device-side wait is bounded (about one second); a wait that runs out, or a
 *     failed device-side check, sets a per-device error word that i8_sync_status()
 *     reports and clears.  The kernels never trap.
 *   - Calls are safe from several host threads on distinct buffers; the error word and
 *     the profiling events below are process-wide.
 */
#ifndef I8LINEAR_H_
#define I8LINEAR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum i8_status {
  I8_OK = 0,
  I8_ERR_INVALID_ARG = 1,  /* bad pointer, shape, threshold or workspace size   */
  I8_ERR_UNSUPPORTED = 2,  /* the current device is not sm_100                  */
  I8_ERR_CUDA = 3,         /* a CUDA runtime call or a launch failed            */
  I8_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out (sync_status)  */
  I8_ERR_DEVICE = 5        /* a device-side consistency check failed            */
} i8_status;

/* Human-readable name of a status code (static storage). */
const char* i8_status_string(i8_status s);

/* After a call returned I8_ERR_CUDA to this host thread: which CUDA runtime or driver call
 * failed and with which error, e.g. "kernel launch failed: cudaErrorInvalidValue (1)".
 * Empty before any such failure; kept until the next one in the same thread.  Thread-local
 * storage owned by the library: valid until this thread's next library call. */
const char* i8_last_error(void);

/*
 * Step 3 -- per-output-channel weight quantisation, run once per weight.
 * Source: "用法" (usage) section -- the weight is quantised when the module moves to the
 * GPU, the codes lie in [-127, 127], and CB * SCB / 127 recovers the fp16 weight; the
 * 64x64 printout there has one absmax per output row.  "内部的 MatMul": the weight is
 * quantised column-wise in the A*B orientation, i.e. per output channel.
 *   W   [N, K] fp16 (read)
 *   CB  [N, K] int8 (written): CB[n,k] = round_half_away(fl32(W[n,k] * fl32(127/SCB[n])))
 *   SCB [N]    fp32 (written): SCB[n]  = max_k |W[n,k]|   (0 for an all-zero row: codes 0)
 * A pure function of W: calling it again on the same W rewrites the same bytes (there is
 * no "quantise twice" state).
 */
i8_status i8_quantize_weight(const void* W, int64_t N, int64_t K, int8_t* CB, float* SCB,
                             void* stream);

/*
 * Step 1 -- outlier column scan.
 * Source: "LLM.int8() 的总结" (outliers are taken column-wise from the hidden states) and
 * "内部的 MatMul" (all outliers of magnitude 6 or larger).
 *   X           [T, K] fp16 (read)
 *   threshold   fp32, not NaN.  Column k is an outlier column when |X[t,k]| >= threshold
 *               for some row t.  threshold <= 0 marks every column; +inf marks only
 *               columns holding an infinity.
 *   col_mask    [ceil(K/32)] uint32 (written; cleared by the call first): column k at
 *               bit k % 32 of word k / 32.
 *   outlier_idx [K] int32 (written): the outlier columns in ascending order, first n_o.
 *   n_outliers  [1] int32 (written): n_o.  Stays on the device; no host copy is made.
 */
i8_status i8_outlier_scan(const void* X, int64_t T, int64_t K, float threshold,
                          uint32_t* col_mask, int32_t* outlier_idx, int32_t* n_outliers,
                          void* stream);

/* Number of fp16 elements of an outlier slice buffer holding `rows` rows:
 * ceil(K/64) * rows * 64.  The slice is stored chunk-major: element (row r, outlier j)
 * sits at ((j / 64) * rows + r) * 64 + j % 64, and entries j >= n_o of the last
 * 64-wide chunk are zero. */
size_t i8_outlier_slice_elems(int64_t rows, int64_t K);

/*
 * Step 2 -- row-wise absmax quantisation of the non-outlier columns of X, and the fp16
 * outlier slice of X.  Source: "absmax 量化" (scale 127/absmax, then multiply and round;
 * the [1.2, -0.5, ..., 5.4] example) and "内部的 MatMul" (hidden states quantised per row).
 *   X           [T, K] fp16 (read)
 *   col_mask, outlier_idx, n_outliers: as written by i8_outlier_scan (read)
 *   Xq          [T, K] int8 (written): outlier columns are 0, the others
 *               round_half_away(fl32(X[t,k] * fl32(127/SCx[t]))) in [-127, 127]
 *   SCx         [T] fp32 (written): max |X[t,k]| over the non-outlier columns (0 if none
 *               is nonzero; then the row's codes are 0)
 *   X_o         fp16 outlier slice, i8_outlier_slice_elems(T, K) elements (written):
 *               X_o(t, j) = X[t, outlier_idx[j]]
 */
i8_status i8_quantize_act(const void* X, int64_t T, int64_t K, const uint32_t* col_mask,
                          const int32_t* outlier_idx, const int32_t* n_outliers, int8_t* Xq,
                          float* SCx, void* X_o, void* stream);

/*
 * Steps 1 and 2 fused: the outlier column scan, the row-wise absmax quantisation and the
 * fp16 outlier slice in ONE launch that reads X from HBM once (each CTA keeps its rows in
 * shared memory across a bounded grid-wide barrier; rows that do not fit are re-read).
 * Sources: as i8_outlier_scan and i8_quantize_act.  Results are identical to
 * i8_outlier_scan followed by i8_quantize_act.
 *   X           [T, K] fp16 (read)            threshold: as in i8_outlier_scan
 *   col_mask    [ceil(K/32) + 1] uint32 (written): the packed mask, then one word of
 *               scratch (the grid barrier); cleared by the call first
 *   outlier_idx [K] int32, n_outliers [1] int32, Xq [T, K] int8, SCx [T] fp32,
 *   X_o         i8_outlier_slice_elems(T, K) fp16: all written, as in the two calls above
 * Uses a cooperative launch of one CTA per SM.
 */
i8_status i8_prepare_act(const void* X, int64_t T, int64_t K, float threshold,
                         uint32_t* col_mask, int32_t* outlier_idx, int32_t* n_outliers,
                         int8_t* Xq, float* SCx, void* X_o, void* stream);

/* Device workspace bytes that i8_linear_forward and i8_igemm_s32 need for these sizes
 * (worst case over the outlier count, which is only known on the device).  0 when a size
 * is invalid. */
size_t i8_linear_workspace_size(int64_t T, int64_t N, int64_t K);

/* The product kernel i8_linear_forward runs for these sizes on the current device (the
 * GEMM variant depends on how many CTA pairs the device holds at once).  Writes one of
 * I8_KERNEL_* to *kind.  I8_ERR_INVALID_ARG for a NULL kind or an invalid size; the
 * device query's error (I8_ERR_CUDA) when the GEMM path needs it and no device answers. */
enum {
  I8_KERNEL_DECODE = 0,     /* decode_kernel: T <= 16 and K <= 65536                  */
  I8_KERNEL_GEMM = 1,       /* i8_gemm_tcgen05_kernel: 256 x 256 tiles per CTA pair   */
  I8_KERNEL_GEMM_WIDE = 2   /* i8_gemm_wide_kernel: 256 x 512 tiles per CTA pair      */
};
i8_status i8_forward_kernel(int64_t T, int64_t N, int64_t K, int32_t* kind);

/*
 * Steps 1, 2, 4, 5 and 6 -- the whole forward of the decomposed linear layer.
 * Sources: "LLM.int8() 的总结" (three steps), "内部的 MatMul" (threshold 6, fp16 outlier
 * product, row/column vector-wise int8 product, dequantise and add), "absmax 量化"
 * (outer-product dequantisation), "用法" (fp16 weights recovered as CB * SCB / 127).
 *   X          [T, K] fp16 (read)         CB [N, K] int8, SCB [N] fp32 (read; from
 *                                         i8_quantize_weight)
 *   bias       [N] fp16 or NULL (read)    threshold: as in i8_outlier_scan
 *   C          [T, N] fp16 (written):
 *     C[t,n] = fp16_rn( (acc[t,n] * SCx[t] / 127 + sum_j X[t,idx_j] * CB[n,idx_j]) * SCB[n] / 127
 *                       + bias[n] )
 *     with acc the exact int32 product of Xq and CB; the outlier sum uses the fp16
 *     operands with fp32 accumulation, and the epilogue runs in fp32.
 *   workspace  device buffer of at least i8_linear_workspace_size(T, N, K) bytes, owned by
 *              the caller; its contents need no initialisation and are scratch after the
 *              call: the decode path drops part of it from the L2 without write-back, so
 *              those bytes may read back as any earlier contents of the memory (calls
 *              sharing one workspace must be ordered on one stream).
 * T <= 16 with K <= 65536 runs the decode path: one kernel (one CTA per SM, each on a
 * K-slice; CB streamed once by TMA into warp-level int8 tensor-core MMAs; steps 1 and 2
 * in its prologue, a cooperative launch when 2*T*K > 128 KB; the outlier sum per K-slice,
 * then across slices, in fp32).  Otherwise: the fused prepare pass and the tcgen05
 * kind::i8 GEMM with the outlier/dequant epilogue (a memset and two kernels).
 */
i8_status i8_linear_forward(const void* X, int64_t T, int64_t K, const int8_t* CB,
                            const float* SCB, const void* bias, int64_t N, float threshold,
                            void* C, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Outlier cache: i8_linear_forward for a serving loop whose outlier columns repeat from
 * call to call.  The blog ("LLM.int8() 的总结"; the emergent-feature discussion) notes that
 * the outliers are systematic: the same few feature dimensions carry them in call after
 * call.  The prefill path's prepare pass gathers the weight's codes in those columns,
 * CB_o (fp16, chunk-major [ceil(n_o/64)][N][64]), on every call; this variant keeps CB_o
 * in a caller-owned cache and skips the gather when a call's outlier set matches the
 * cached one.  The output is bit-identical to i8_linear_forward's.
 *
 * i8_outlier_cache_size(N, K, max_cols): bytes of a cache that holds up to max_cols
 * outlier columns (rounded up to a multiple of 64, at most K rounded up) of an [N, K]
 * weight: a header (8 words and the ceil(K/32) mask words, padded to 256 B) plus
 * N * 128 bytes per 64 columns.  Returns 0 for invalid arguments (N or K <= 0, K % 16 != 0,
 * max_cols <= 0).  Host-only arithmetic.
 *
 * i8_outlier_cache_reset(cache, cache_bytes, stream): marks the cache empty (clears its
 * header's first 8 words on `stream`).  Call it once on a new cache -- its memory starts
 * undefined -- and again whenever the weight's codes CB change in place; the cache is keyed
 * by the outlier set, N, K and the CB device pointer, not by CB's contents.  Returns
 * I8_ERR_INVALID_ARG for a NULL or unaligned cache or cache_bytes < 32, I8_ERR_CUDA if the
 * memset cannot be enqueued.
 *
 * i8_linear_forward_cached(X, T, K, CB, SCB, bias, N, threshold, C, workspace,
 *                          workspace_bytes, cache, cache_bytes, stream):
 *   every argument but the last three exactly as in i8_linear_forward (the workspace is
 *   still needed, of the same size);
 *   cache        device buffer, 16-byte aligned, owned by the caller, reset once before its
 *                first use; cache_bytes its size, which sets its capacity in columns
 *                (at least one 64-column chunk: i8_outlier_cache_size(N, K, 64)).
 * The prepare pass decides on the device, with no host synchronisation: when the cache is
 * valid and holds this call's exact outlier set for the same CB pointer, N and K, the GEMM
 * reads CB_o from the cache and nothing is gathered; when the set differs (and n_o fits
 * the capacity), CB_o is gathered into the cache, which is then keyed by this set; when
 * n_o exceeds the capacity, CB_o is gathered into the workspace and the cache is left as
 * it was.  Decode batches (T <= 16, K <= 65536) take the decode kernel, which needs no
 * CB_o, and leave the cache untouched.  Calls sharing one cache must be ordered on one
 * stream.  A call that fails on the device (I8_ERR_TIMEOUT from i8_sync_status) leaves the
 * cache either as it was or empty, never keyed to a partly written slice.  Returns I8_ERR_INVALID_ARG, with nothing launched, for a NULL or unaligned
 * cache, a capacity below 64 columns, or any argument i8_linear_forward rejects.
 */
size_t i8_outlier_cache_size(int64_t N, int64_t K, int64_t max_cols);
i8_status i8_outlier_cache_reset(void* cache, size_t cache_bytes, void* stream);
i8_status i8_linear_forward_cached(const void* X, int64_t T, int64_t K, const int8_t* CB,
                                   const float* SCB, const void* bias, int64_t N,
                                   float threshold, void* C, void* workspace,
                                   size_t workspace_bytes, void* cache, size_t cache_bytes,
                                   void* stream);

/*
 * FP8 (e4m3) variant of the layer.  The blog names 8-bit floating point only as the next
 * step after int8 (its closing outlook); these calls take the plainest reading of it:
 * every step above is kept, and the int8 absmax code is replaced by an e4m3 code of the
 * same scaled value --
 *   scale s = fl32(448 / absmax)   (448 = the largest finite e4m3 magnitude),
 *   code    = e4m3 rounding of fl32(x * s): nearest, ties to even, beyond 448 saturating,
 * with 448 in place of 127 in both dequantisations:
 *   C[t,n] = fp16_rn( (acc[t,n] * SCx[t] / 448 + sum_j X[t,idx_j] * dec(CB[n,idx_j]))
 *                     * SCB[n] / 448 + bias[n] ),
 * acc being the e4m3 x e4m3 product accumulated in fp32 by the tensor cores
 * (tcgen05 kind::f8f6f4).  e4m3 is the "fn" format of the OCP 8-bit floating-point
 * specification (1 sign, 4 exponent bits with bias 7, 3 fraction bits, no infinities).
 * Codes are stored one byte each (uint8_t), row-major, like the int8 codes.
 *
 * i8_quantize_weight_e4m3(W, N, K, CB, SCB, stream): as i8_quantize_weight, with CB [N, K]
 *   e4m3 codes.
 * i8_prepare_act_e4m3(...): as i8_prepare_act, with Xq [T, K] e4m3 codes (outlier columns
 *   code 0).
 * i8_linear_workspace_size_e4m3(T, N, K): workspace bytes of i8_linear_forward_e4m3 (0 for
 *   invalid shapes).
 * i8_linear_forward_e4m3(X, T, K, CB, SCB, bias, N, threshold, C, workspace,
 *   workspace_bytes, stream): the e4m3 forward; arguments as in i8_linear_forward, with CB
 *   from i8_quantize_weight_e4m3 and a workspace of i8_linear_workspace_size_e4m3 bytes.
 *   Every T takes the fused prepare pass and the tensor-core GEMM (there is no separate
 *   decode kernel for this variant).
 * Errors as for the int8 calls.
 */
i8_status i8_quantize_weight_e4m3(const void* W, int64_t N, int64_t K, uint8_t* CB, float* SCB,
                                  void* stream);
i8_status i8_prepare_act_e4m3(const void* X, int64_t T, int64_t K, float threshold,
                              uint32_t* col_mask, int32_t* outlier_idx, int32_t* n_outliers,
                              uint8_t* Xq, float* SCx, void* X_o, void* stream);
size_t i8_linear_workspace_size_e4m3(int64_t T, int64_t N, int64_t K);
i8_status i8_linear_forward_e4m3(const void* X, int64_t T, int64_t K, const uint8_t* CB,
                                 const float* SCB, const void* bias, int64_t N, float threshold,
                                 void* C, void* workspace, size_t workspace_bytes, void* stream);

/*
 * i8_linear_forward without a workspace argument: the same forward as i8_linear_forward,
 * with its scratch taken from a fixed 32 MiB array that the library itself holds in
 * device memory.  The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory and have none to lend -- for example a plugin inside a
 * host application that owns every device allocation and hands its plugins no scratch,
 * or a serving loop that must never call cudaMalloc/cudaFree, because those calls can
 * synchronise the whole device and stall other work.  This call allocates nothing.
 *   X, T, K, CB, SCB, bias, N, threshold, C, stream: exactly as in i8_linear_forward.
 * Limit: sizes whose i8_linear_workspace_size(T, N, K) exceeds 32 MiB are rejected with
 * I8_ERR_INVALID_ARG before anything is launched (decode batches of large layers, e.g.
 * T <= 16 with N = 57344, K = 14336, fit; large prefill shapes do not).
 * Every GPU that loads the library holds the 32 MiB until the process exits.  The first
 * call on a device looks up the array's device address (once per device, with that
 * device current); make that first call before any stream capture.  All calls share the
 * one array and it keeps the last call's contents; nothing in it needs to start at zero
 * (each call clears what it uses).  Calls that overlap on the GPU -- on different
 * streams, or from different host threads -- race on the array: order them on one stream.
 */
i8_status i8_linear_forward_noalloc(const void* X, int64_t T, int64_t K, const int8_t* CB,
                                    const float* SCB, const void* bias, int64_t N,
                                    float threshold, void* C, void* stream);

/*
 * Backward of the fp16-weight training mode.  Source: "用法" (usage) -- a layer built with
 * has_fp16_weights=True keeps its fp16 weights for int8/fp16 mixed-precision training and
 * re-quantises them for every forward; CB * SCB / 127 recovers the weight.  The blog gives
 * no gradient formulas; these calls take the plainest reading, the backward of
 * y = x W^T + b passed straight through the quantisation:
 *
 * i8_linear_backward_input(dY, T, N, W, K, dX, stream):
 *   dX[T, K] = dY[T, N] * W[N, K]             (dY, W, dX fp16; W may be the fp16 weight
 *                                             or the dequantised weight below)
 * i8_linear_backward_weight(dY, X, T, N, K, dW, stream):
 *   dW[N, K] = dY[T, N]^T * X[T, K]           (dY, X, dW fp16)
 *   Both on the tcgen05 tensor cores (kind::f16): fp16 products summed in fp32, one
 *   round-to-nearest-even to fp16 at the end.  W and X are read in their stored layout
 *   (row-major [N, K] and [T, K]); the tensor cores take them as MN-major operands.
 * i8_bias_grad(dY, T, N, db, stream):
 *   db[N] = fp16(sum_t dY[t, n]), summed in fp32 in a fixed order (deterministic).
 * i8_dequantize_weight(CB, SCB, N, K, W, stream):
 *   W[n, k] = fp16_rn(fl32(CB[n, k] * fl32(SCB[n] / 127)))   (W fp16 [N, K], written)
 * i8_dequantize_weight_e4m3(CB, SCB, N, K, W, stream):
 *   the same with e4m3 codes: their values times fl32(SCB[n] / 448).
 *
 * Shapes: T, N, K > 0, K % 16 == 0, and N % 8 == 0 for the three calls that read dY (its
 * row pitch must be a multiple of 16 bytes for TMA).  Every pointer is a 16-byte aligned
 * device pointer owned by the caller; outputs are written in full.  Violations return
 * I8_ERR_INVALID_ARG with nothing launched; errors otherwise as for the forward.
 */
i8_status i8_linear_backward_input(const void* dY, int64_t T, int64_t N, const void* W,
                                   int64_t K, void* dX, void* stream);
i8_status i8_linear_backward_weight(const void* dY, const void* X, int64_t T, int64_t N,
                                    int64_t K, void* dW, void* stream);
i8_status i8_bias_grad(const void* dY, int64_t T, int64_t N, void* db, void* stream);
i8_status i8_dequantize_weight(const int8_t* CB, const float* SCB, int64_t N, int64_t K, void* W,
                               void* stream);
i8_status i8_dequantize_weight_e4m3(const uint8_t* CB, const float* SCB, int64_t N, int64_t K,
                                    void* W, void* stream);

/*
 * Step 4 alone -- acc[T, N] int32 = A[T, K] int8 * B[N, K]^T int8, on the same kernels
 * as i8_linear_forward (the tcgen05 GEMM, or the decode kernel for T <= 16 and
 * K <= 65536), with the epilogue writing the raw accumulator.  Source: "内部的 MatMul" (the 8-bit matrix
 * multiplication).  Exact: |acc| <= K * 127^2 must fit in int32 (K <= 133144).
 *   workspace: at least i8_linear_workspace_size(T, N, K) bytes.
 */
i8_status i8_igemm_s32(const int8_t* A, int64_t T, int64_t K, const int8_t* B, int64_t N,
                       int32_t* acc, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Synchronise `stream`, then read and clear the per-device error word.
 * Returns I8_ERR_CUDA if the stream reports an error, I8_ERR_TIMEOUT if a bounded wait
 * ran out, I8_ERR_DEVICE if a device-side check failed, else I8_OK.
 */
i8_status i8_sync_status(void* stream);

/*
 * Benchmark hook: when both are non-NULL cudaEvent_t handles, every following
 * i8_linear_forward records `start` just before and `stop` just after its dominant
 * kernel (the GEMM; on the decode path the decode kernel, i.e. the whole forward), on the
 * call's stream.  NULL, NULL turns it off.
 * Process-wide; meant for single-threaded benchmarking.
 */
i8_status i8_set_profile_events(void* start_event, void* stop_event);

/*
 * Failure-path self test: launch one thread that waits on a device barrier nothing will
 * complete, with a wait limit of `limit_ns` nanoseconds (1e3 .. 1e10).  The wait runs
 * out, the error word is set, and the kernel returns; a following i8_sync_status()
 * must give I8_ERR_TIMEOUT.  Faults nothing and leaves the context usable.
 */
i8_status i8_selftest_bounded_wait(int64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* I8LINEAR_H_ */

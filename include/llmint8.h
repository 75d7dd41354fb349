/*
 * llmint8.h - C ABI of the B200 (sm_100a) LLM.int8() mixed-precision decomposed linear layer
 *
 *   Y[M, N] = X[M, K] . W^T,  W stored as int8 CB[N, K] + fp32 per-output-channel absmax SCB[N]
 *
 * The method (LLM.int8(), Dettmers et al.): split the feature columns of X into "outlier"
 * columns (some entry with |x| >= threshold, default 6) and regular columns; multiply the
 * outlier part in fp16 against the matching fp16 weights; quantize the regular part
 * vector-wise (one absmax per row of X, one per output channel of W), multiply in int8 with
 * int32 accumulation, dequantize by the outer product of the two absmax vectors / 127^2 and
 * add the two parts in fp16.  Sources: "A gentle introduction to 8-bit matrix multiplication
 * for transformers at scale" (Hugging Face blog, zh translation), sections 模型量化介绍,
 * LLM.int8() 温和总结, MatMul 内部 and 用法; "LLM.int8(): 8-Bit Matrix Multiplication for
 * Transformers at Scale" (azimuth.plus summary), sections الابتكار الأول, الابتكار الثاني and
 * الصورة الكاملة.
 *
 * Conventions for every call
 *   - fp16 tensors are IEEE binary16 bit patterns (uint16_t); all tensors are dense and
 *     row-major (last index contiguous).
 *   - Every tensor pointer is a DEVICE pointer (cudaMalloc / torch CUDA memory) on the
 *     current device and 16-byte aligned.  The caller owns every buffer; the library never
 *     allocates or frees device memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are asynchronous
 *     on that stream: the returned status covers argument checks and launch errors only.
 *     Conditions found on the device (outlier capacity exceeded, a bounded wait that timed
 *     out) are written to the status word of the workspace; read them with
 *     llmint8_device_status().  Each call that takes a workspace overwrites that word.
 *   - Shapes: M >= 1; K and N are multiples of 16 and >= 16; K <= 131072 (so that
 *     |C| <= K * 127^2 < 2^31).  Violations return LLMINT8_ERR_UNSUPPORTED_SHAPE.
 *   - No C++ exception crosses this interface.
 */
#ifndef LLMINT8_H
#define LLMINT8_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define LLMINT8_API __attribute__((visibility("default")))
#else
#define LLMINT8_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    LLMINT8_OK = 0,
    LLMINT8_ERR_INVALID_ARG = 1,         /* null or misaligned pointer, NaN threshold, ... */
    LLMINT8_ERR_UNSUPPORTED_SHAPE = 2,   /* shape outside the rules above */
    LLMINT8_ERR_WORKSPACE_TOO_SMALL = 3, /* ws_bytes below the matching *_workspace_size() */
    LLMINT8_ERR_OUTLIER_CAPACITY = 4,    /* (device) more outlier columns than the capacity */
    LLMINT8_ERR_TIMEOUT = 5,             /* (device) a bounded wait in a kernel gave up */
    LLMINT8_ERR_CUDA = 6,                /* a CUDA runtime call or launch failed */
    LLMINT8_ERR_DEVICE_CHECK = 7         /* (device, debug build only) a bounds check failed */
} llmint8_status;

/*
 * Weight quantization, once per layer.  The blog quantizes the weight per column of the
 * logical K x N weight, i.e. per output channel (section MatMul 内部); CB and SCB are the
 * names of section 用法.
 *   W   fp16 [N, K]  input, nn.Linear layout (row n = output channel n).
 *   CB  int8 [N, K]  output: CB[n,k] = round_half_even(fl32(W[n,k] * fl32(127 / SCB[n]))).
 *   SCB fp32 [N]     output: SCB[n] = max_k |W[n,k]| (0 gives an all-zero row).
 * Pure function of W: calling it twice gives identical bytes.
 */
LLMINT8_API llmint8_status llmint8_quantize_weight_colwise(const uint16_t *W, int64_t N, int64_t K,
                                               int8_t *CB, float *SCB, void *stream);

/*
 * Outlier-column detection and row-wise quantization of the activations (the first
 * steps of the method: outlier features are the columns of the hidden state holding a
 * value of magnitude >= threshold; hidden states are quantized by row).
 *   X           fp16 [M, K] input.
 *   threshold   |x| >= threshold marks column j an outlier; +inf allowed (no outliers),
 *               <= 0 marks every column; NaN -> LLMINT8_ERR_INVALID_ARG.
 *   Xq          int8 [M, K] output; outlier columns hold 0.
 *   SCA         fp32 [M] output: absmax of row i over the regular columns (0 if none / all 0).
 *   outlier_idx int32 [cap] output: the outlier columns in ascending order (first `cap`).
 *   n_outliers  int32 [1] output (device): the true number of outlier columns.
 *   cap         capacity of outlier_idx (0 <= cap <= K).  n_outliers > cap sets the device
 *               status LLMINT8_ERR_OUTLIER_CAPACITY (Xq and SCA stay exact).
 *   ws          device workspace of llmint8_quantize_workspace_size(M, K) bytes.
 */
LLMINT8_API llmint8_status llmint8_quantize_rows_and_find_outliers(const uint16_t *X, int64_t M, int64_t K,
                                                       float threshold, int8_t *Xq, float *SCA,
                                                       int32_t *outlier_idx, int32_t *n_outliers,
                                                       int64_t cap, void *ws, size_t ws_bytes,
                                                       void *stream);

LLMINT8_API size_t llmint8_quantize_workspace_size(int64_t M, int64_t K);

/*
 * The decomposed linear layer (the whole method: outlier columns -> fp16 product against
 * the matching fp16 weight rows; the rest -> vector-wise int8 product with int32
 * accumulation, dequantized by the outer product SCA_i * SCB_n / 127^2; the two summed
 * into the fp16 output).
 *   X       fp16 [M, K] input activations.
 *   CB, SCB int8 [N, K], fp32 [N] from llmint8_quantize_weight_colwise.
 *   bias    fp16 [N] or NULL.
 *   W_fp16  fp16 [N, K] or NULL.  NULL (inference, weights kept only in int8): the fp16
 *           weights of the outlier columns are fp16(fl32(fl32(CB * SCB) / 127)).
 *           Non-NULL: the original fp16 weights are used for the outlier columns.
 *   threshold   as in llmint8_quantize_rows_and_find_outliers.
 *   max_outliers capacity for outlier columns, 0 <= max_outliers <= K; it sizes the
 *           workspace.  More outlier columns than this sets LLMINT8_ERR_OUTLIER_CAPACITY in
 *           the device status (the output is then incomplete but memory stays in bounds).
 *   Y       fp16 [M, N] output: fp16(C*SCA_i*SCB_n/127^2 + sum_{j in O} X[i,j]*W_o[n,j] + bias_n),
 *           evaluated in fp32 with int32 C.
 *   ws      device workspace of llmint8_linear_workspace_size(M, N, K, max_outliers) bytes.
 *   C_debug int32 [M, N] or NULL: when given, also receives the exact int8 accumulators C.
 * Kernels (int8 codes, outlier columns and C do not depend on the choice; Y may differ in
 * the last fp32 rounding): M <= 16, K <= 16384, threshold > 0 and max_outliers <= 256 run one
 * kernel whose first CTAs quantize X (each a slice of the columns) while the others stream
 * the weight through tcgen05 MMAs.  Other shapes run
 * outlier detection, row quantization (with the gather of the outlier weight rows) and a
 * persistent tcgen05 GEMM, on CTA pairs when M > 128.  Kernels of a call are launched as
 * programmatic dependents: each may start while the work before it on the stream finishes,
 * and waits for that work before it reads or writes global memory.
 */
LLMINT8_API llmint8_status llmint8_linear(const uint16_t *X, int64_t M, int64_t K, const int8_t *CB,
                              const float *SCB, int64_t N, const uint16_t *bias,
                              const uint16_t *W_fp16, float threshold, int64_t max_outliers,
                              uint16_t *Y, void *ws, size_t ws_bytes, void *stream,
                              int32_t *C_debug);

LLMINT8_API size_t llmint8_linear_workspace_size(int64_t M, int64_t N, int64_t K, int64_t max_outliers);

/*
 * llmint8_linear_next_bitmaps: llmint8_linear that also finds, while it writes Y, the outlier
 * columns of a next layer that takes Y as its input X.  Outliers are found per feature column
 * of a layer's input (blog section LLM.int8() 温和总结, step 1), so for that layer they are
 * the columns of Y where some row reaches its threshold; forming them here saves the next
 * call the pass over its input that llmint8_linear makes to find them.  X, M, K, CB, SCB, N,
 * bias, W_fp16, threshold, max_outliers, Y, ws, ws_bytes, stream and C_debug, and every
 * result, are as for llmint8_linear.  Then:
 *   next_threshold  the next layer's threshold (rules as in
 *                   llmint8_quantize_rows_and_find_outliers: <= 0 marks every column; NaN ->
 *                   LLMINT8_ERR_INVALID_ARG).
 *   next_bitmaps    uint32 [ceil(M/32)][ceil(N/32)], device, 4-byte aligned, owned by the
 *                   caller, fully overwritten: bit (n % 32) of word [b][n / 32] is set iff some
 *                   row m of the 32-row block b (32 b <= m < min(M, 32 b + 32)) has
 *                   |Y[m, n]| >= next_threshold, Y as stored (fp16).  Give them to the next
 *                   layer's llmint8_linear_with_bitmaps with n_bitmaps = ceil(M/32).
 * The GEMM path forms each word in the epilogue that writes those values of Y (an OR over a
 * warp's 32 rows; no atomics); on the decode path each warp owns its output columns' bits of
 * the words they straddle (and the bits past N) and writes them with an atomic AND, then an
 * atomic OR, so nothing needs clearing first.
 */
LLMINT8_API llmint8_status llmint8_linear_next_bitmaps(const uint16_t *X, int64_t M, int64_t K,
                                           const int8_t *CB, const float *SCB, int64_t N,
                                           const uint16_t *bias, const uint16_t *W_fp16,
                                           float threshold, int64_t max_outliers, uint16_t *Y,
                                           void *ws, size_t ws_bytes, void *stream,
                                           int32_t *C_debug, float next_threshold,
                                           uint32_t *next_bitmaps);

/*
 * Token-parallel (M-split) layers.  When the rows of X are split over ranks, the outlier set
 * must still be that of the whole X: an outlier column is one where ANY row reaches the
 * threshold (blog section LLM.int8() 温和总结: outliers are found per feature column of the
 * whole hidden state), so a rank's own rows do not decide it.  Each rank computes its
 * rows' bitmap, the ranks exchange the bitmaps (an all-gather of ceil(K/32) words each), and
 * every rank runs the layer on its rows with the OR of all of them.  The rows it gets are
 * llmint8_linear's int8 codes and int32 C for those rows of the whole X, and Y within the
 * layer's tolerance (the same bytes when the same kernel serves both: the decode kernel for
 * at most 16 rows, the GEMM otherwise; the two may round the last fp32 step differently).
 *
 * llmint8_outlier_bitmap: bit (j % 32) of bitmap[j / 32] is set iff some row of X [M, K]
 *   has |X[i, j]| >= threshold (threshold rules as in
 *   llmint8_quantize_rows_and_find_outliers).  bitmap: uint32 [ceil(K/32)], device, 4-byte
 *   aligned, fully overwritten.  ws: llmint8_quantize_workspace_size(M, K) bytes; its device
 *   status is LLMINT8_OK after the call (every column is listed internally, so no capacity
 *   applies).
 */
LLMINT8_API llmint8_status llmint8_outlier_bitmap(const uint16_t *X, int64_t M, int64_t K,
                                      float threshold, uint32_t *bitmap, void *ws,
                                      size_t ws_bytes, void *stream);

/*
 * llmint8_linear_with_bitmaps: llmint8_linear with the outlier set given instead of found:
 *   O = the columns set in ANY of the n_bitmaps bitmaps [n_bitmaps][ceil(K/32)] (uint32,
 *   device, 4-byte aligned; 1 <= n_bitmaps <= 65536).  Bits at columns >= K are ignored.
 *   Every other argument, the workspace (llmint8_linear_workspace_size(M, N, K,
 *   max_outliers)) and the output are as for llmint8_linear, without a threshold.  Shapes of
 *   the decode path (M <= 16, K <= 16384, max_outliers <= 256) run the decode kernel with the
 *   merged bitmaps as its outlier set; others run the outlier compaction, the row
 *   quantization and the tcgen05 GEMM.  More outlier columns than max_outliers sets
 *   LLMINT8_ERR_OUTLIER_CAPACITY in the device status.
 */
LLMINT8_API llmint8_status llmint8_linear_with_bitmaps(const uint16_t *X, int64_t M, int64_t K,
                                           const int8_t *CB, const float *SCB, int64_t N,
                                           const uint16_t *bias, const uint16_t *W_fp16,
                                           const uint32_t *bitmaps, int64_t n_bitmaps,
                                           int64_t max_outliers, uint16_t *Y, void *ws,
                                           size_t ws_bytes, void *stream, int32_t *C_debug);

/*
 * llmint8_linear on HOST activations and outputs (a calling convenience with no counterpart
 * on the pages: the layer itself is llmint8_linear).  On `stream`, in order: copy X_host
 * [M, K] fp16 into the device buffer X_dev, run llmint8_linear(X_dev -> Y_dev), copy Y_dev
 * [M, N] fp16 into Y_host.  No C_debug output.
 *   X_host, Y_host  HOST pointers owned by the caller.  Page-locked (cudaHostAlloc /
 *                   torch pin_memory) memory keeps the call asynchronous; pageable memory
 *                   works, but CUDA then copies synchronously.  Y_host holds the output only
 *                   after the stream has reached the end of the call (synchronize it).
 *   X_dev, Y_dev    DEVICE buffers of M*K and M*N fp16 values, owned by the caller, 16-byte
 *                   aligned; they hold X and Y afterwards.
 *   CB, SCB, bias, W_fp16, threshold, max_outliers, ws, ws_bytes: as for llmint8_linear.
 * Every argument check of llmint8_linear runs before the first copy, with the same codes;
 * a NULL host pointer returns LLMINT8_ERR_INVALID_ARG.  A failed copy returns
 * LLMINT8_ERR_CUDA.  Conditions found on the device go to the workspace's status word.
 */
LLMINT8_API llmint8_status llmint8_linear_host(const uint16_t *X_host, int64_t M, int64_t K,
                                   const int8_t *CB, const float *SCB, int64_t N,
                                   const uint16_t *bias, const uint16_t *W_fp16,
                                   float threshold, int64_t max_outliers, uint16_t *Y_host,
                                   uint16_t *X_dev, uint16_t *Y_dev, void *ws, size_t ws_bytes,
                                   void *stream);

/*
 * Weight dequantization W_out[n,k] = fp16(fl32(fl32(CB[n,k] * SCB[n]) / 127)) (blog
 * section 用法: the fp16 weights are recovered as (CB * SCB) / 127).
 */
LLMINT8_API llmint8_status llmint8_dequant(const int8_t *CB, const float *SCB, int64_t N, int64_t K,
                               uint16_t *W_out, void *stream);

/*
 * Synchronizes `stream` and returns the device status word of a workspace used by the
 * last llmint8_linear / llmint8_quantize_rows_and_find_outliers call on it
 * (LLMINT8_OK, LLMINT8_ERR_OUTLIER_CAPACITY, LLMINT8_ERR_TIMEOUT or, in the debug build,
 * LLMINT8_ERR_DEVICE_CHECK), or LLMINT8_ERR_CUDA.
 * The result is meaningful only for a workspace that at least one call has used; a
 * zero-filled one reads LLMINT8_OK.
 */
LLMINT8_API llmint8_status llmint8_device_status(const void *ws, void *stream);

/* Also returns the device outlier count of a llmint8_linear workspace (synchronizes). */
LLMINT8_API llmint8_status llmint8_workspace_outlier_count(const void *ws, void *stream, int32_t *count);

/*
 * Read-back of the fp16 outlier-weight rows W_o that the last llmint8_linear or
 * llmint8_linear_with_bitmaps call on `ws` multiplied X's outlier columns with (blog section
 * 用法: the fp16 weights are recovered as (CB * SCB) / 127; with W_fp16 given, the original
 * fp16 weights): W_o[n, j] = fp16(fl32(fl32(CB[n, O_j] * SCB[n]) / 127)), or W_fp16[n, O_j],
 * for the outlier columns O_0 < O_1 < ... of that call.  It lets a test compare this step of
 * the layer bit for bit.
 *   ws            the workspace of that call.
 *   M, N, K, max_outliers  that call's arguments (they fix where W_o lies in the workspace).
 *   Wo            DEVICE fp16 [N, n_cols], row-major, 16-byte aligned, owned by the caller.
 *   n_cols        0 <= n_cols <= max_outliers; columns past that call's outlier count hold 0.
 * The GEMM path keeps W_o in the workspace on every call.  The decode path forms it in
 * registers and stores it into the workspace only when the call was given C_debug; after a
 * decode-path call without C_debug the result is undefined.  Asynchronous on `stream` (one
 * device-to-device copy); LLMINT8_ERR_INVALID_ARG for a bad pointer or n_cols,
 * LLMINT8_ERR_UNSUPPORTED_SHAPE for shapes llmint8_linear rejects.
 */
LLMINT8_API llmint8_status llmint8_workspace_outlier_weights(const void *ws, int64_t M, int64_t N,
                                                 int64_t K, int64_t max_outliers,
                                                 uint16_t *Wo, int64_t n_cols, void *stream);

/* Static English text for a status code. */
LLMINT8_API const char *llmint8_status_string(llmint8_status status);

/*
 * Build flags of the loaded library: bit 0 is set in the debug build (libllmint8_debug.so,
 * compiled with LLMINT8_DEBUG).  There the kernels also check, on the device, that every
 * outlier column index they list or read is below K, that no more than the capacity are
 * listed, and that every tile they store lies inside its output; a failed check records
 * LLMINT8_ERR_DEVICE_CHECK in the workspace's device status (read with
 * llmint8_device_status) and the kernel carries on without trapping.  Results are otherwise
 * the release build's, bit for bit.
 */
LLMINT8_API int llmint8_build_flags(void);

/*
 * Upper bound, in nanoseconds, of every wait inside the GEMM and decode kernels of later calls
 * (process-wide; default 1e9).  A wait that runs out records LLMINT8_ERR_TIMEOUT in the
 * device status and the kernel winds down and returns.  Tests set a tiny bound to
 * exercise that path.  ns == 0 restores the default.
 */
LLMINT8_API llmint8_status llmint8_set_wait_timeout_ns(uint64_t ns);

/*
 * Measurement hooks (no counterpart on the pages; they let a benchmark time the product
 * kernel of a call with CUDA events and count launches):
 *   llmint8_set_profile_events(start, stop): two cudaEvent_t.  While both are non-NULL,
 *     every llmint8_linear, llmint8_linear_next_bitmaps, llmint8_linear_with_bitmaps and
 *     llmint8_linear_noalloc call records `start` on its stream immediately before its
 *     product kernel (the GEMM; on the decode path, the decode kernel) and `stop`
 *     immediately after it.  NULL, NULL disables.
 *     Process-wide; the caller owns the events and must keep them alive while set.
 *   llmint8_kernel_launch_count(): number of kernels this library has launched in the
 *     process so far.
 */
LLMINT8_API llmint8_status llmint8_set_profile_events(void *start, void *stop);
LLMINT8_API uint64_t llmint8_kernel_launch_count(void);

/*
 * llmint8_linear without a workspace argument.  The paper has no counterpart: this is a
 * calling convenience.  It is for callers that cannot allocate device memory where they
 * call the layer: a token-by-token decode loop that must not call cudaMalloc/cudaFree
 * between steps (cudaFree waits for the whole device), or a plain C host without a device
 * allocator of its own.  The call allocates nothing.  Its scratch - the 256-byte header that
 * receives the call's status words and outlier count - is a fixed device array inside this
 * library, one per device.
 *   Arguments X, M, K, CB, SCB, N, bias, W_fp16, threshold, max_outliers, Y, stream: as
 *     for llmint8_linear (same layouts, same output, the same bytes).  There is no C_debug
 *     output.  Profile events set with llmint8_set_profile_events are recorded around its
 *     kernel as for llmint8_linear.
 *   Covered shapes are those of the decode path: M <= 16, K <= 16384 (K, N multiples of
 *     16), threshold > 0 and max_outliers <= 256.  Anything larger returns
 *     LLMINT8_ERR_UNSUPPORTED_SHAPE before any CUDA call; use llmint8_linear there.
 *   scratch_out  NULL, or receives the device address of the calling device's scratch, the
 *     same 256-byte header as at the start of an llmint8_linear workspace.  So
 *     llmint8_device_status(*scratch_out, stream) and
 *     llmint8_workspace_outlier_count(*scratch_out, ...) report the device status and the
 *     outlier count of the last call on that device.
 *   Set-up: the first call on each device looks up the scratch's address
 *     (cudaGetSymbolAddress, with the device current), which may load this library's
 *     device code.  Make that first call before any stream capture.  The address is kept for
 *     the life of the process: a device reset (cudaDeviceReset) between calls is not
 *     supported.
 *   Nothing in the scratch needs clearing between calls: each call tags its status words
 *     with a fresh call number and stores the outlier count.
 *   Calls on one stream, in order, are safe.  Calls that overlap on one device (two
 *     streams, or host threads without stream order between them) share its scratch and
 *     race on it: their outputs are unaffected, but the status and count read back may
 *     belong to either call.
 * Returns LLMINT8_ERR_INVALID_ARG for NULL or misaligned pointers (16 bytes) or a NaN
 * threshold, and LLMINT8_ERR_CUDA if the set-up or a launch fails.
 */
LLMINT8_API llmint8_status llmint8_linear_noalloc(const uint16_t *X, int64_t M, int64_t K,
                                      const int8_t *CB, const float *SCB, int64_t N,
                                      const uint16_t *bias, const uint16_t *W_fp16,
                                      float threshold, int64_t max_outliers, uint16_t *Y,
                                      void *stream, void **scratch_out);

#ifdef __cplusplus
}
#endif

#endif /* LLMINT8_H */

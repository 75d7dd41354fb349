// Internal launch interface between the C ABI (api.cu) and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>

#include "common.cuh"

namespace llmint8 {

// Adds n to the process-wide count of kernels launched by the library.
void note_launches(int n);

// Row-split plan of the outlier scan: the columns are covered by `col_blocks` CTAs of
// 256 threads x 8 columns, the rows by `splits` ranges of `rows_per_split` rows.
struct ScanPlan {
    int64_t col_blocks = 0, splits = 0, rows_per_split = 0, nwords = 0;
};
ScanPlan scan_plan(int64_t M, int64_t K);

cudaError_t launch_outlier_detect(const __half *X, int64_t M, int64_t K, float threshold,
                                  const ScanPlan &plan, uint32_t *partial, uint32_t *bitmap,
                                  int32_t *idx, int64_t cap, int32_t *count, StatusRef status,
                                  cudaStream_t s);
// The outlier set as the OR of n_bitmaps caller-supplied column bitmaps [n][ceil(K/32)]
// (bits at columns >= K ignored): merged bitmap, ascending list (first cap), count, status.
cudaError_t launch_outlier_merge(const uint32_t *bitmaps, int64_t n_bitmaps, int64_t K,
                                 uint32_t *bitmap, int32_t *idx, int64_t cap, int32_t *count,
                                 StatusRef status, cudaStream_t s);
// Row quantization of X (and, with Wo non-null, the gather of the outlier weights Wo
// [N, xo_pitch] from CB/SCB or W16, in the same launch).  The scan, compaction and this
// kernel are programmatic dependents of whatever precedes them in the stream.
cudaError_t launch_quantize_rows(const __half *X, int64_t M, int64_t K, const uint32_t *bitmap,
                                 const int32_t *idx, const int32_t *count, int64_t cap,
                                 int64_t xo_pitch, int8_t *Xq, float *SCA, __half *Xo,
                                 const int8_t *CB, const float *SCB, const __half *W16, int64_t N,
                                 __half *Wo, cudaStream_t s);
cudaError_t launch_quantize_weight(const __half *W, int64_t N, int64_t K, int8_t *CB, float *SCB,
                                   cudaStream_t s);
cudaError_t launch_dequant(const int8_t *CB, const float *SCB, int64_t N, int64_t K,
                           __half *W_out, cudaStream_t s);

// The tcgen05 GEMM with the fused fp16 outlier product and dequantizing epilogue.
struct GemmLaunch {
    const int8_t *Xq;        // [M, K]
    const int8_t *CB;        // [N, K]
    const __half *Xo;        // [M, pitch]   (may be null when cap == 0)
    const __half *Wo;        // [N, pitch]
    int64_t pitch;           // columns of Xo / Wo (multiple of 64)
    const int32_t *count;    // device outlier count
    int64_t cap;             // capacity (columns usable in Xo / Wo)
    const float *SCA;        // [M]
    const float *SCB;        // [N]
    const __half *bias;      // [N] or null
    __half *Y;               // [M, N]
    int32_t *C_debug;        // [M, N] or null
    StatusRef status;
    int64_t M, N, K;
    uint64_t timeout_ns;
};
cudaError_t launch_gemm(const GemmLaunch &g, cudaStream_t s);

}  // namespace llmint8

namespace llmint8 {

// Decode path (M <= kDecodeMaxM, K <= kDecodeMaxK): a cluster of CTAs quantizes X into a
// ready-to-copy image of the tensor-core operand plus small tables in the workspace; the
// weight-streaming tcgen05 kernel, launched as its programmatic dependent, starts streaming
// CB at once and waits for that image only before its first MMA.
constexpr int kDecodeMaxM = 16;
constexpr int kDecodeMaxK = 8192;
constexpr int kDecodeMaxOutliers = 256;

// Written by the decode quantize kernel, copied whole into every decode CTA.
struct DecodeTables {
    unsigned long long ready;                 // call epoch, stored last (release)
    int32_t n_out;                            // outlier columns used (<= capacity)
    int32_t pad;
    float sca[kDecodeMaxM];                   // row absmax over the regular columns
    int32_t idx[kDecodeMaxOutliers];          // outlier columns, ascending
};
static_assert(sizeof(DecodeTables) % 16 == 0, "copied with a bulk copy");

// Bytes of the quantized-X operand image: 16 rows x K rounded up to 128, in 128-column
// blocks of two 1024-byte swizzled 8-row atoms.
__host__ __device__ constexpr int64_t decode_image_bytes(int64_t K) {
    return kDecodeMaxM * ((K + 127) / 128 * 128);
}

struct DecodeLaunch {
    const __half *X;         // [M, K]
    const int8_t *CB;        // [N, K]
    const float *SCB;        // [N]
    const __half *W16;       // [N, K] or null
    const __half *bias;      // [N] or null
    __half *Y;               // [M, N]
    int32_t *C_debug;        // [M, N] or null
    __half *Wo;              // [N, wo_pitch] or null: receives the outlier weights used
    int64_t wo_pitch;
    int32_t *count;          // device outlier count (workspace header)
    uint8_t *image;          // workspace: decode_image_bytes(K), 1024-byte aligned
    DecodeTables *tables;    // workspace
    StatusRef status;
    int64_t M, N, K, cap;
    float threshold;
    uint64_t timeout_ns;
};
cudaError_t launch_decode(const DecodeLaunch &d, cudaStream_t s);

}  // namespace llmint8

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
    uint32_t *ybits;         // [ceil(M/32)][ceil(N/32)] outlier bitmaps of Y for the next
                             // layer (|Y| >= ythreshold per column and 32-row block), or null
    float ythreshold;
    StatusRef status;
    int64_t M, N, K;
    uint64_t timeout_ns;
};
cudaError_t launch_gemm(const GemmLaunch &g, cudaStream_t s);

}  // namespace llmint8

namespace llmint8 {

// Decode path (M <= kDecodeMaxM, K <= kDecodeMaxK, at most kDecodeMaxOutliers outlier
// columns): one weight-streaming tcgen05 kernel per call.  Its first CTAs quantize X (each a
// slice of the columns; they exchange their partial row maxima and outlier counts) and publish
// the outlier columns, row scales and the int8 operand image through a DecodeTable and the
// image in the workspace; every other CTA streams a band of weight rows.
constexpr int kDecodeMaxM = 16;
constexpr int kDecodeMaxK = 16384;
constexpr int kDecodeMaxOutliers = 256;

// What the quantizer CTAs publish (workspace, 256-byte aligned).
//   part[q][m]  (call << 32) | fp32 bits of quantizer q's row-m maximum of |x| over the regular
//               columns of its slice (m < kDecodeMaxM), then (call << 32) | the number of
//               outlier columns in its slice: one 64-bit store each, so a word that carries
//               the call's number carries its value;
//   done[q]     the call's number, stored with release semantics once quantizer q's k-blocks of
//               the operand image and its entries of idx are written (quantizer 0: also sca,
//               total and n_out).
constexpr int kDecodeMaxQuantizers = 8;
struct DecodeTable {
    unsigned long long done[kDecodeMaxQuantizers];
    unsigned long long part[kDecodeMaxQuantizers][kDecodeMaxM + 1];
    int32_t total;                            // outlier columns found
    int32_t n_out;                            // ... of them listed (<= capacity)
    float sca[kDecodeMaxM];                   // row absmax over the regular columns
    int32_t idx[kDecodeMaxOutliers];          // outlier columns, ascending
};

// Bytes of the int8 operand image the quantizer writes: one block of 16 rows (8 when M <= 8)
// x 128 bytes per 128-column k-block.
__host__ __device__ constexpr int64_t decode_image_bytes(int64_t M, int64_t K) {
    return (K + 127) / 128 * (M <= 8 ? 8 : kDecodeMaxM) * 128;
}

// Launch geometry of the decode kernel for one shape.
struct DecodePlan {
    int Rt = 0;              // weight rows (output channels) per tile
    int tiles = 0, grid = 0, kblocks = 0;
    int rows = 0;            // rows of an operand-image block (8 or 16)
    int stages = 0, smem = 0;
    int inflight = 0;        // weight stages a streamer keeps on their way at most
    int nq = 0;              // quantizer CTAs (the first nq of the grid)
    int bpq = 0;             // k-blocks per quantizer
    int nst = 0;             // weight stages per tile (2 k-blocks each)
    int nistage = 0;         // operand-image stages of a streamer
    bool resident = false;   // ... holding every k-block (filled once)
    uint32_t tail_off = 0, xo_off = 0, ring_off = 0;
};
DecodePlan decode_plan(int64_t M, int64_t N, int64_t K, int64_t cap, int sms);

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
    const uint32_t *bitmaps; // [n_bitmaps][ceil(K/32)]: the outlier set given, or null
    int64_t n_bitmaps;
    uint32_t *ybits;         // [ceil(N/32)]: outlier bitmap of Y for the next layer, or null
    float ythreshold;
    int32_t *count;          // device outlier count (workspace header)
    DecodeTable *table;      // workspace
    uint8_t *image;          // workspace: decode_image_bytes(M, K), 1024-byte aligned
    StatusRef status;
    int64_t M, N, K, cap;
    float threshold;
    uint64_t timeout_ns;
};
cudaError_t launch_decode(const DecodeLaunch &d, cudaStream_t s);

}  // namespace llmint8

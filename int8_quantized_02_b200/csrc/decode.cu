// Decode path of the LLM.int8() layer (few activation rows, M <= 16).
//
// At decode sizes the layer is bound by streaming the int8 weight CB from HBM once, and
// everything else must hide under that stream.  Two kernels:
//
// llmint8_decode_quantize_kernel (one cluster of 8 CTAs x 1024 threads) quantizes X once:
//   one thread per (row, 8-column chunk), each warp holding all 16 rows of two chunks, CTA r
//   of the cluster 1/8 of the columns.  The outlier bits of a chunk (|x| >= threshold in any
//   row) are an OR across 16 lanes; the row maxima over the regular columns reduce in
//   registers, across warps, and across the cluster through distributed shared memory
//   (one hardware cluster barrier); the int8 codes go into the workspace as a byte-exact
//   image of the tensor-core operand (16 rows, 128-byte swizzled K-major blocks, outlier
//   columns and padding 0), next to a table of SCA and the ascending outlier columns.  It
//   lets its dependent launch as soon as the work before it in the stream is complete.
//
// llmint8_decode_kernel (one CTA per 128-row weight tile, programmatic dependent launch):
//   warp 0        TMA producer: streams 128-row x 128-byte tiles of CB (16 KB) through a ring
//                 of shared-memory stages from its first cycle - it needs nothing from X - and
//                 asks L2 for the rest of its first tile as well, so that HBM keeps streaming
//                 while the MMA waits for the quantized X (every weight byte is still read
//                 from HBM once per call; the later stage loads find it in L2);
//   warp 1        waits until the quantize kernel publishes (an acquire on the call epoch it
//                 stores last), bulk-copies the operand image and the table into shared
//                 memory, then issues tcgen05.mma kind::i8
//                 with the weight tile as the 128-row operand and the quantized X as the
//                 16-column operand: D[n, m] = sum_k CB[n, k] Xq[m, k] into a 128 x 16 int32
//                 TMEM accumulator (double-buffered over tiles);
//   warps 4..7    epilogue: while the weights stream, each thread (one output row n) builds
//                 sum_{j in O} X[m, O_j] * W_o[n, O_j] + bias_n (the fp16 outlier part of the
//                 decomposition, weights from the bytes of the outlier columns) and its scale;
//                 after the tile's last MMA: D -> registers, y = D * SCA_m * SCB_n / 127^2 +
//                 that part -> fp16.
// Same method and rounding as the GEMM path (LLM.int8() summary, sections الابتكار الثاني
// and الصورة الكاملة; blog sections MatMul 内部 and 用法).  Every wait is bounded.
#include <cudaTypedefs.h>

#include <cstddef>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace llmint8 {

namespace {

constexpr int DM = kDecodeMaxM;         // activation rows held (MMA N)
constexpr int DBM = 128;                // weight rows per tile (MMA M)
constexpr int DBK = 128;                // bytes of K per stage
constexpr int DSTAGE = DBM * DBK;       // 16 KB
constexpr int DTHREADS = 256;
constexpr int DMAX_STAGES = 12;
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in per CTA
constexpr int QTHREADS = 1024;          // quantize kernel: one cluster of QCL CTAs
constexpr int QWARPS = QTHREADS / 32;
constexpr int QCL = 8;
// chunk pairs (16 columns) per warp: K <= kDecodeMaxK keeps every item in registers
constexpr int QKEEP = (kDecodeMaxK / 16 / QCL + QWARPS - 1) / QWARPS;
// k-blocks of a CTA's first tile requested into L2 ahead of the stage ring, so that HBM keeps
// streaming while the first MMA waits for the quantized X
constexpr int kPrefetchBlocks = 64;
// Independent int32 accumulators per tile: k-block it accumulates into sub-accumulator
// it % DSUB, so consecutive MMAs do not wait on each other's result (a 128 x 16 MMA is too
// short to hide the accumulate dependency); the epilogue adds them (exact in int32).
constexpr int DSUB = 4;
constexpr uint32_t DTMEM_COLS = 2 * DSUB * kDecodeMaxM;   // double-buffered over tiles

__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __half22float2(h[e]);
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}

// Byte offset of Xq[m, k0 ..] (k0 a multiple of 8) in the 128-byte-swizzled K-major layout:
// per 128-column block, `rows` (16, or 8 when M <= 8) rows of 128 bytes in 8-row atoms of
// 1024 bytes; the 16-byte chunk index within a row is XORed with (row mod 8).  With 8 rows
// the MMA's second 8-row group is one shared all-zero atom after the last block (see
// image_desc), so the image takes half the shared memory and the weight ring two more stages.
__device__ __forceinline__ uint32_t xq_offset(int m, int k0, int rows) {
    const int kb = k0 >> 7, c = k0 & 127;
    return (uint32_t)(kb * (rows * 128) + (m >> 3) * 1024 + (m & 7) * 128 +
                      ((((c >> 4) ^ (m & 7)) << 4) | (c & 15)));
}

__host__ __device__ constexpr int image_rows(int M) { return M <= 8 ? 8 : kDecodeMaxM; }
// Bytes of the image: the blocks, plus the shared zero atom when it has 8 rows.
__host__ __device__ constexpr int image_bytes(int kblocks, int rows) {
    return kblocks * rows * 128 + (rows == 8 ? 1024 : 0);
}

// Descriptor of the image's block at `saddr` (+ k offset) for the 16-column MMA operand: the
// two 8-row groups are `sbo` bytes apart (1024 in the 16-row image; in the 8-row image the
// distance to the zero atom, so that rows 8..15 read as zeros).
__device__ __forceinline__ uint64_t image_desc(uint32_t saddr, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);      // start address / 16
    d |= (uint64_t)1u << 16;                      // leading byte offset (unused, 16 B)
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;  // stride byte offset between 8-row groups
    d |= (uint64_t)1u << 46;                      // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                      // swizzle: 128 B
    return d;
}

__device__ __forceinline__ uint32_t outlier_bits(const float *f, float threshold) {
    uint32_t b = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) b |= (fabsf(f[e]) >= threshold ? 1u : 0u) << e;
    return b;
}

__device__ __forceinline__ float masked_max(const float *f, uint32_t skip, float r) {
#pragma unroll
    for (int e = 0; e < 8; ++e)
        if (!((skip >> e) & 1u)) r = fmaxf(r, fabsf(f[e]));
    return r;
}

// Eight absmax-quantized int8 codes, packed little-endian; a set bit in `skip` gives 0.
__device__ __forceinline__ uint2 quant8(const float *f, float mul, uint32_t skip) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        int q = 0;
        if (!((skip >> e) & 1u)) q = max(-127, min(127, __float2int_rn(__fmul_rn(f[e], mul))));
        const uint32_t b = (uint32_t)(q & 0xff);
        if (e < 4) lo |= b << (8 * e);
        else hi |= b << (8 * (e - 4));
    }
    return make_uint2(lo, hi);
}

struct QArgs {
    const __half *X;
    int M, K, cap;
    float threshold;
    uint8_t *image;
    DecodeTables *tables;
    int32_t *count;
    StatusRef status;
    unsigned long long epoch;
    int rows;                                // image rows: 16, or 8 when M <= 8
};

// One cluster of QCL CTAs.  CTA r owns the chunk pairs [r*PP, (r+1)*PP); one thread per
// (row, chunk) item, its values kept in registers between the two passes.
__global__ void __launch_bounds__(QTHREADS, 1) llmint8_decode_quantize_kernel(const QArgs a) {
    // launched as a programmatic dependent of whatever precedes it in the stream: wait for it
    // before touching X or the workspace, then let the weight-streaming kernel launch
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    __shared__ float part[QCL][DM];          // row maxima of every CTA of the cluster
    __shared__ uint32_t pmax[DM];            // this CTA's (float bits, >= 0: int order)
    __shared__ float mult[DM];
    __shared__ uint8_t flags_all[kDecodeMaxK / 8];   // CTA 0: outlier bits of every chunk
    const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
    const int m = lane & 15;                 // the row this thread handles
    const int half = lane >> 4;              // which chunk of the warp's pair
    const uint32_t r = cluster_ctarank();
    const int nchunks = a.K / 8;
    const int npairs = nchunks / 2;          // K is a multiple of 16
    const int pp = (npairs + QCL - 1) / QCL;
    const int p0 = (int)r * pp, p1 = min(npairs, p0 + pp);
    const uint4 *X4 = reinterpret_cast<const uint4 *>(a.X);

    uint4 v[QKEEP];
#pragma unroll
    for (int i = 0; i < QKEEP; ++i) {
        const int p = p0 + warp + i * QWARPS;
        v[i] = (p < p1 && m < a.M) ? __ldg(X4 + (int64_t)m * nchunks + 2 * p + half)
                                   : make_uint4(0, 0, 0, 0);
    }
    if (t < DM) pmax[t] = 0u;
    __syncthreads();

    // pass 1: outlier bits of each chunk (OR over its 16 lanes = rows), published to CTA 0;
    // row maxima over the regular columns
    uint32_t fl[QKEEP];
    float rm = 0.0f;
    const uint32_t flags0 = map_to_rank(smem_addr(flags_all), 0);
#pragma unroll
    for (int i = 0; i < QKEEP; ++i) {
        fl[i] = 0;
        const int p = p0 + warp + i * QWARPS;
        if (p < p1) {                        // uniform over the warp
            float f[8];
            unpack8(v[i], f);
            uint32_t b = outlier_bits(f, a.threshold);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) b |= __shfl_xor_sync(0xffffffffu, b, o);
            fl[i] = b;
            if (m == 0) st_cluster_u8(flags0 + (uint32_t)(2 * p + half), b);
            rm = masked_max(f, b, rm);
        }
    }
    rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, 16));
    if (half == 0 && m < a.M && rm > 0.0f) atomicMax(&pmax[m], __float_as_uint(rm));
    __syncthreads();
    if (t < DM) {
        const uint32_t dst = smem_addr(&part[r][t]);
        for (int rr = 0; rr < QCL; ++rr) st_cluster_u32(map_to_rank(dst, (uint32_t)rr), pmax[t]);
    }
    // every CTA's flags and partial maxima are in place after this
    cluster_barrier_all();

    if (t < DM) {
        float amax = 0.0f;
        for (int rr = 0; rr < QCL; ++rr) amax = fmaxf(amax, part[rr][t]);
        mult[t] = (t < a.M && amax > 0.0f) ? __fdiv_rn(127.0f, amax) : 0.0f;
        if (r == 0) a.tables->sca[t] = amax;
    }
    __syncthreads();

    // pass 2: every (row, chunk) of this CTA into the operand image; rows >= M, all-zero rows
    // and outlier columns are written as 0
    const float mul = mult[m];
#pragma unroll
    for (int i = 0; i < QKEEP; ++i) {
        const int p = p0 + warp + i * QWARPS;
        if (p < p1) {
            const int c = 2 * p + half;
            uint2 q = make_uint2(0, 0);
            if (mul > 0.0f) {
                float f[8];
                unpack8(v[i], f);
                q = quant8(f, mul, fl[i]);
            }
            if (m < a.rows) *reinterpret_cast<uint2 *>(a.image + xq_offset(m, c * 8, a.rows)) = q;
        }
    }
    // every CTA's part of the image is written before CTA 0 publishes it
    __threadfence();
    __syncwarp();
    cluster_barrier_all();
    if (r != 0) return;   // nothing of this CTA is read by its peers any more

    // CTA 0: padding columns of the image (and its zero atom), ascending outlier list, count,
    // status
    const int kpad_chunks = (a.K + 127) / 128 * 16;
    for (int i = t; i < (kpad_chunks - nchunks) * a.rows; i += QTHREADS) {
        const int c = nchunks + i / a.rows, mm = i % a.rows;
        *reinterpret_cast<uint2 *>(a.image + xq_offset(mm, c * 8, a.rows)) = make_uint2(0, 0);
    }
    if (a.rows == 8 && t < 128)
        reinterpret_cast<uint2 *>(a.image + (kpad_chunks / 16) * 1024)[t] = make_uint2(0, 0);
    if (warp == 0) {
        const int per = (nchunks + 31) / 32;
        const int c0 = lane * per, c1 = min(nchunks, c0 + per);
        int cnt = 0;
        for (int c = c0; c < c1; ++c) cnt += __popc(flags_all[c]);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int pos = incl - cnt;
        for (int c = c0; c < c1; ++c) {
            uint32_t b = flags_all[c];
            while (b) {
                const int e = __ffs(b) - 1;
                b &= b - 1;
                if (pos < a.cap) a.tables->idx[pos] = c * 8 + e;
                ++pos;
            }
        }
        const int total = __shfl_sync(0xffffffffu, incl, 31);
        if (lane == 0) {
            a.tables->n_out = min(total, a.cap);
            *a.count = total;
            a.status.set(total > a.cap ? LLMINT8_ERR_OUTLIER_CAPACITY : LLMINT8_OK);
        }
    }
    // publish: the image and table are complete (the dependent kernel bulk-copies them)
    __threadfence();
    fence_proxy_async_global();
    __syncthreads();
    if (t == 0)
        asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(&a.tables->ready), "l"(a.epoch)
                     : "memory");
}

struct DTail {
    uint64_t full[DMAX_STAGES];
    uint64_t empty[DMAX_STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint64_t xbar;                       // operand image and table have landed
    uint32_t tmem_base;
    int abort_flag;
    alignas(16) DecodeTables tab;
    alignas(16) __half xo[kDecodeMaxOutliers * DM];   // X at the outlier columns, [j][m]
};
static_assert(offsetof(DTail, tab) % 16 == 0, "the table is a bulk-copy destination");
static_assert(offsetof(DTail, xbar) % 8 == 0, "mbarriers are 8-byte aligned");

struct DArgs {
    unsigned long long epoch;
    const __half *X;
    const int8_t *CB;
    const float *SCB;
    const __half *W16;
    const __half *bias;
    __half *Y;
    int32_t *C_debug;
    __half *Wo;                          // [N, wo_pitch] or null
    int64_t wo_pitch;
    const uint8_t *image;
    const DecodeTables *tables;
    StatusRef status;
    int M, N, K;
    int stages;
    int kblocks;
    int tiles;
    uint32_t xq_off;                     // byte offsets in shared memory
    uint32_t tail_off;
    uint64_t timeout_ns;
    int rows;                            // image rows: 16, or 8 when M <= 8
};

__global__ void __launch_bounds__(DTHREADS, 1)
llmint8_decode_kernel(const __grid_constant__ CUtensorMap tmCB, const DArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DTail *tail = reinterpret_cast<DTail *>(smem + a.tail_off);
    uint8_t *xq = smem + a.xq_off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int S = a.stages;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&tail->full[s]), 1);
            mbar_init(smem_addr(&tail->empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&tail->acc_full[s]), 1);
            mbar_init(smem_addr(&tail->acc_empty[s]), 4);
        }
        mbar_init(smem_addr(&tail->mma_done), 1);
        mbar_init(smem_addr(&tail->xbar), 1);
        tail->abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmCB);
    }
    if (warp == 1) tmem_alloc(smem_addr(&tail->tmem_base), DTMEM_COLS);
    // the next call's first kernel may launch now (it waits for this grid before it reads)
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const BoundedWait wait{&tail->abort_flag, a.status, a.timeout_ns};

    if (warp == 0) {
        // --------------------------------------------------- weight stream (TMA) ----
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, used = 0, last_parity = 0;
            for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
                const int n0 = tile * DBM;
                for (int it = 0; it < a.kblocks; ++it) {
                    const int kb = rotated_kblock(it, tile, a.kblocks);
                    if (tile == (int)blockIdx.x && it == S) {
                        // the ring is full: request the rest of this first tile into L2
                        const int last = min(a.kblocks, S + kPrefetchBlocks);
                        for (int pf = S; pf < last; ++pf)
                            tma_prefetch_l2_2d(&tmCB, rotated_kblock(pf, tile, a.kblocks) * DBK,
                                               n0);
                    }
                    if (!wait(smem_addr(&tail->empty[stage]), phase ^ 1)) goto drain;
                    const uint32_t full = smem_addr(&tail->full[stage]);
                    mbar_arrive_expect_tx(full, DSTAGE);
                    tma_load_2d(smem_addr(smem + stage * DSTAGE), &tmCB, kb * DBK, n0, full);
                    used |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        drain:
            for (int s = 0; s < S; ++s)
                if (used & (1u << s))
                    drain_wait(smem_addr(&tail->full[s]), (last_parity >> s) & 1u, a.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issue ----
        if (lane == 0) {
            // the quantize kernel (already running: this grid is its programmatic dependent)
            // publishes the image with a release store of the call's epoch
            bool published = false;
            {
                const uint64_t t0 = global_timer_ns();
                for (uint32_t it = 0;; ++it) {
                    unsigned long long v;
                    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];"
                                 : "=l"(v)
                                 : "l"(&a.tables->ready)
                                 : "memory");
                    if (v == a.epoch) {
                        published = true;
                        break;
                    }
                    if ((it & 63u) == 0u && (tail->abort_flag ||
                                             global_timer_ns() - t0 > a.timeout_ns)) {
                        tail->abort_flag = 1;
                        a.status.timed_out();
                        break;
                    }
                }
            }
            fence_proxy_async_global();
            const uint32_t xbar = smem_addr(&tail->xbar);
            const uint32_t img_bytes = (uint32_t)image_bytes(a.kblocks, a.rows);
            mbar_arrive_expect_tx(xbar, img_bytes + (uint32_t)sizeof(DecodeTables));
            bulk_load_1d(smem_addr(xq), a.image, img_bytes, xbar);
            bulk_load_1d(smem_addr(&tail->tab), a.tables, (uint32_t)sizeof(DecodeTables), xbar);
            const bool have_x = published && wait(xbar, 0);
            const uint32_t idesc = idesc_i8(DBM, DM);
            const uint32_t xq_base = smem_addr(xq);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; have_x && tile < a.tiles; tile += gridDim.x) {
                if (!wait(smem_addr(&tail->acc_empty[acc]), acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * DSUB * DM);
                bool good = true;
                for (int it = 0; it < a.kblocks; ++it) {
                    const int kb = rotated_kblock(it, tile, a.kblocks);
                    if (!wait(smem_addr(&tail->full[stage]), phase)) {
                        good = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + stage * DSTAGE);
                    const uint32_t sb = xq_base + (uint32_t)(kb * a.rows * 128);
                    const uint32_t sbo =
                        a.rows == 8 ? (uint32_t)((a.kblocks - kb) * 1024) : 1024u;
                    const uint32_t dsub = d + (uint32_t)((it % DSUB) * DM);
#pragma unroll
                    for (int k = 0; k < DBK / 32; ++k)
                        mma_i8(dsub, sw128_desc(sa + 32 * k), image_desc(sb + 32 * k, sbo), idesc,
                               (it >= DSUB) || k != 0);
                    tc_commit(smem_addr(&tail->empty[stage]));
                    if (++stage == S) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!good) break;
                tc_commit(smem_addr(&tail->acc_full[acc]));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            if (!have_x) drain_wait(xbar, 0, a.status);   // the copies land before exit
            tc_commit(smem_addr(&tail->mma_done));
            drain_wait(smem_addr(&tail->mma_done), 0, a.status);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ epilogue ----
        // Everything of an output row except the int8 product - its scale, bias and fp16
        // outlier part - is computed while the MMAs still stream the weights; after the last
        // MMA of a tile only the accumulator read, one FMA per value and the stores remain.
        const int qd = warp & 3;
        const int et = threadIdx.x - 128;                 // 0..127 over the epilogue warps
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        const float inv = 1.0f / 16129.0f;
        int okx = 0;
        if (lane == 0) okx = wait(smem_addr(&tail->xbar), 0) ? 1 : 0;   // the table is in
        okx = __shfl_sync(0xffffffffu, okx, 0);
        const int n_out = okx ? tail->tab.n_out : 0;
        // X at the outlier columns (an input of the call, complete before this grid launched)
        for (int i = et; i < n_out * DM; i += 128) {
            const int j = i / DM, mm = i % DM;
            tail->xo[i] = mm < a.M ? a.X[(int64_t)mm * a.K + tail->tab.idx[j]]
                                   : __float2half_rn(0.0f);
        }
        named_barrier(1, 128);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; okx && tile < a.tiles; tile += gridDim.x) {
            const int n = tile * DBM + qd * 32 + lane;
            const bool live = n < a.N;
            float o[DM];
            float scale = 0.0f;
#pragma unroll
            for (int m = 0; m < DM; ++m) o[m] = 0.0f;
            if (live) {
                const float sb = a.SCB[n];
                const float b = a.bias ? __half2float(a.bias[n]) : 0.0f;
                scale = sb * inv;
                const int8_t *cbrow = a.CB + (int64_t)n * a.K;
                for (int j = 0; j < n_out; ++j) {
                    const int col = tail->tab.idx[j];
                    const __half wh = a.W16 ? a.W16[(int64_t)n * a.K + col]
                                            : __float2half_rn(__fdiv_rn(
                                                  __fmul_rn((float)cbrow[col], sb), 127.0f));
                    if (a.Wo) a.Wo[(int64_t)n * a.wo_pitch + j] = wh;
                    const float w = __half2float(wh);
                    const uint4 *xv = reinterpret_cast<const uint4 *>(tail->xo + j * DM);
                    float f0[8], f1[8];
                    unpack8(xv[0], f0);
                    unpack8(xv[1], f1);
#pragma unroll
                    for (int m = 0; m < 8; ++m) {
                        o[m] = fmaf(f0[m], w, o[m]);
                        o[m + 8] = fmaf(f1[m], w, o[m + 8]);
                    }
                }
#pragma unroll
                for (int m = 0; m < DM; ++m) o[m] += b;
            }
            int okw = 0;
            if (lane == 0) okw = wait(smem_addr(&tail->acc_full[acc]), acc_phase) ? 1 : 0;
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!okw) break;
            tc_fence_after();
            uint32_t d[DM];
            tmem_ld_32x16(tl + (uint32_t)(acc * DSUB * DM), d);
            for (int u = 1; u < DSUB; ++u) {
                if (u >= a.kblocks) break;               // sub-accumulators never written
                uint32_t e[DM];
                tmem_ld_32x16(tl + (uint32_t)((acc * DSUB + u) * DM), e);
                tmem_wait_ld();
#pragma unroll
                for (int m = 0; m < DM; ++m) d[m] += e[m];
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&tail->acc_empty[acc]));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
            if (live) {
#pragma unroll
                for (int m = 0; m < DM; ++m) {
                    if (m < a.M) {
                        const float y = fmaf((float)(int32_t)d[m], tail->tab.sca[m] * scale, o[m]);
                        a.Y[(int64_t)m * a.N + n] = __float2half_rn(y);
                        if (a.C_debug) a.C_debug[(int64_t)m * a.N + n] = (int32_t)d[m];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, DTMEM_COLS);
    }
}

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

}  // namespace

cudaError_t launch_decode(const DecodeLaunch &d, cudaStream_t s) {
    static std::mutex mu;
    static int sms_cache[64] = {0};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int sms;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (sms_cache[dev] == 0) {
            int n = 0;
            err = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
            if (err != cudaSuccess) return err;
            err = cudaFuncSetAttribute(llmint8_decode_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_LIMIT);
            if (err != cudaSuccess) return err;
            sms_cache[dev] = n;
        }
        sms = sms_cache[dev];
    }

    // 1. quantize X once (one CTA)
    QArgs q;
    q.X = d.X;
    q.M = (int)d.M;
    q.K = (int)d.K;
    q.cap = (int)d.cap;
    q.threshold = d.threshold;
    q.image = d.image;
    q.tables = d.tables;
    q.count = d.count;
    q.status = d.status;
    q.epoch = d.status.tag >> 4;
    q.rows = image_rows((int)d.M);
    {
        cudaLaunchConfig_t qc = {};
        cudaLaunchAttribute qa[2];
        qa[0].id = cudaLaunchAttributeClusterDimension;
        qa[0].val.clusterDim.x = QCL;
        qa[0].val.clusterDim.y = 1;
        qa[0].val.clusterDim.z = 1;
        qa[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        qa[1].val.programmaticStreamSerializationAllowed = 1;
        qc.gridDim = dim3(QCL);
        qc.blockDim = dim3(QTHREADS);
        qc.dynamicSmemBytes = 0;
        qc.stream = s;
        qc.attrs = qa;
        qc.numAttrs = 2;
        err = cudaLaunchKernelEx(&qc, llmint8_decode_quantize_kernel, q);
        note_launches(1);
        if (err != cudaSuccess) return err;
    }

    // 2. the weight-streaming product, allowed to start before step 1 finishes
    DArgs a;
    a.epoch = d.status.tag >> 4;
    a.X = d.X;
    a.CB = d.CB;
    a.SCB = d.SCB;
    a.W16 = d.W16;
    a.bias = d.bias;
    a.Y = d.Y;
    a.C_debug = d.C_debug;
    a.Wo = d.Wo;
    a.wo_pitch = d.wo_pitch;
    a.image = d.image;
    a.tables = d.tables;
    a.status = d.status;
    a.M = (int)d.M;
    a.N = (int)d.N;
    a.K = (int)d.K;
    a.kblocks = (int)ceil_div(d.K, DBK);
    a.tiles = (int)ceil_div(d.N, DBM);
    a.timeout_ns = d.timeout_ns;
    // shared memory: [stages][quantized X][tail], 1024-byte aligned pieces
    a.rows = image_rows((int)d.M);
    const int xq_bytes = (int)align_up(image_bytes(a.kblocks, a.rows), 1024);
    const int tail_bytes = (int)align_up(sizeof(DTail), 1024);
    const int room = SMEM_LIMIT - 1024 - xq_bytes - tail_bytes;
    a.stages = std::min(DMAX_STAGES, room / DSTAGE);
    if (a.stages < 2) return cudaErrorInvalidValue;
    a.xq_off = (uint32_t)(a.stages * DSTAGE);
    a.tail_off = a.xq_off + (uint32_t)xq_bytes;
    const int smem = (int)(a.tail_off + sizeof(DTail) + 1024);
    if (smem > SMEM_LIMIT) return cudaErrorInvalidValue;

    auto enc = encoder();
    if (!enc) return cudaErrorInvalidValue;
    CUtensorMap tm;
    cuuint64_t dims[2] = {(cuuint64_t)d.K, (cuuint64_t)d.N};
    cuuint64_t strides[1] = {(cuuint64_t)d.K};
    cuuint32_t box[2] = {DBK, DBM};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(d.CB), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    // QCL SMs stay with the quantize kernel while this grid starts
    cfg.gridDim = dim3((unsigned)std::min(a.tiles, std::max(1, sms - QCL)));
    cfg.blockDim = dim3(DTHREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, llmint8_decode_kernel, tm, a);
    note_launches(1);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace llmint8

// Decode path of the LLM.int8() layer (few activation rows, M <= 16).
//
// At decode sizes the layer is bound by streaming the int8 weight CB from HBM once, and the
// rest must hide under that stream.  One cooperative kernel (every CTA resident, one per SM),
// one CTA of 512 threads per 128-row weight tile (grid-stride when there are more tiles):
//
//   all warps     first quantize X together, with no weight traffic in flight (weight requests
//                 issued earlier queue in front of X's loads and of the exchanges through the
//                 scratch, and that costs more than it overlaps).  CTA g owns 1/G of the columns: one lane per (row,
//                 8-column chunk), each warp holding all 16 rows of two chunks, so the outlier
//                 bits of a chunk (|x| >= threshold in any row) are an OR across 16 lanes and
//                 the row maxima over the regular columns reduce in registers.  Outlier bits
//                 and partial maxima go to workspace scratch; after a grid barrier every CTA
//                 has SCA and the ascending outlier set, quantizes its columns and writes the
//                 int8 codes into a byte image of the tensor-core operand (16 rows, 128-byte
//                 swizzled K-major blocks, outlier columns and padding 0); after a second
//                 grid barrier every CTA bulk-copies the whole image into shared memory;
//   warp 0 lane 0 TMA producer: then streams 128-row x 128-byte tiles of CB (16 KB) through
//                 a ring of shared-memory stages (enough in flight to keep HBM busy);
//   warp 1        tcgen05.mma kind::i8 with the weight tile as the 128-row operand and the
//                 quantized X as the 16-column operand: D[n, m] = sum_k CB[n, k] Xq[m, k] into
//                 a 128 x 16 int32 TMEM accumulator (double-buffered over tiles);
//   warps 4..7    epilogue: D -> registers; y = D * SCA_m * SCB_n / 127^2
//                 + sum_{j in O} X[m, O_j] * W_o[n, O_j] + bias_n (the fp16 outlier part of
//                 the decomposition, weights from the bytes of the outlier columns) -> fp16.
// Same method and rounding as the GEMM path (LLM.int8() summary, sections الابتكار الثاني
// and الصورة الكاملة; blog sections MatMul 内部 and 用法).  Every wait is bounded; the grid
// barriers use a fixed bound and no atomics, so every CTA always reaches both.
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
constexpr int DTHREADS = 512;
constexpr int DWARPS = DTHREADS / 32;
constexpr int DMAX_STAGES = 12;
constexpr int DCAP = kDecodeMaxOutliers;
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in per CTA
constexpr int QKEEP = 4;                // chunk pairs per warp kept in registers

struct DTail {
    uint64_t full[DMAX_STAGES];
    uint64_t empty[DMAX_STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint64_t xbar;                       // the operand image has landed
    uint32_t tmem_base;
    int abort_flag;
    int n_out;                           // outlier columns used (<= cap)
    int bar_ok;
    uint32_t rowmax[DM];                 // float bits (non-negative: int order == float order)
    float sca[DM];
    float mult[DM];                      // fl32(127 / sca), 0 for rows >= M or all-zero rows
    int warp_tot[DWARPS];
    int32_t idx[DCAP];                   // outlier columns (ascending)
    alignas(16) __half xo[DCAP * DM];    // X at the outlier columns, [j][m] (read as uint4)
};
static_assert(offsetof(DTail, xo) % 16 == 0, "xo is read with 16-byte loads");
static_assert(offsetof(DTail, xbar) % 8 == 0, "mbarriers are 8-byte aligned");

struct DArgs {
    const __half *X;
    const int8_t *CB;
    const float *SCB;
    const __half *W16;
    const __half *bias;
    __half *Y;
    int32_t *C_debug;
    int32_t *count;
    DecodeScratch *scr;
    uint8_t *image;
    StatusRef status;
    unsigned long long epoch;
    int M, N, K, cap;
    float threshold;
    int stages;
    int kblocks;
    int tiles;
    uint32_t xq_off;                     // byte offsets in shared memory
    uint32_t tail_off;
    uint64_t timeout_ns;
};

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
// per 128-column block, 16 rows of 128 bytes in two 8-row atoms of 1024 bytes; the 16-byte
// chunk index within a row is XORed with (row mod 8).
__device__ __forceinline__ uint32_t xq_offset(int m, int k0) {
    const int kb = k0 >> 7, c = k0 & 127;
    return (uint32_t)(kb * (DM * 128) + (m >> 3) * 1024 + (m & 7) * 128 +
                      ((((c >> 4) ^ (m & 7)) << 4) | (c & 15)));
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

// Barrier over every CTA of the (cooperative, all-resident) grid, without atomics: CTA g
// publishes the call's epoch in arrived[g] (release), then one thread per peer waits
// (acquire) until that peer's word carries the epoch.  Words left by earlier calls hold
// older epochs, so the scratch needs no initialization.  Bounded by a fixed limit.
__device__ __forceinline__ void grid_barrier(unsigned long long *arrived, unsigned long long epoch,
                                             DTail *tail, StatusRef status) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(arrived + blockIdx.x),
                     "l"(epoch)
                     : "memory");
    }
    if (threadIdx.x < gridDim.x) {
        constexpr uint64_t kLimitNs = 1000000000ull;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t it = 0;; ++it) {
            unsigned long long v;
            asm volatile("ld.acquire.gpu.global.u64 %0, [%1];"
                         : "=l"(v)
                         : "l"(arrived + threadIdx.x)
                         : "memory");
            if (v == epoch) break;
            if ((it & 63u) == 0u && global_timer_ns() - t0 > kLimitNs) {
                status.timed_out();
                tail->bar_ok = 0;
                break;
            }
        }
    }
    __syncthreads();
}

__global__ void __launch_bounds__(DTHREADS, 1)
llmint8_decode_kernel(const __grid_constant__ CUtensorMap tmCB, const DArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DTail *tail = reinterpret_cast<DTail *>(smem + a.tail_off);
    uint8_t *xq = smem + a.xq_off;
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int S = a.stages;
    const int m = lane & 15;                 // quantization: the row this lane handles
    const int half = lane >> 4;              //               which chunk of the warp's pair
    const int nchunks = a.K / 8;
    const int npairs = nchunks / 2;          // K is a multiple of 16
    const int pp = (npairs + (int)gridDim.x - 1) / (int)gridDim.x;
    const int p0 = (int)blockIdx.x * pp, p1 = min(npairs, p0 + pp);   // this CTA's pairs
    const uint4 *X4 = reinterpret_cast<const uint4 *>(a.X);

    // this CTA's columns of X first, ahead of every weight request
    uint4 keep[QKEEP];
#pragma unroll
    for (int i = 0; i < QKEEP; ++i) {
        const int p = p0 + warp + i * DWARPS;
        keep[i] = (p < p1 && m < a.M) ? __ldg(X4 + (int64_t)m * nchunks + 2 * p + half)
                                      : make_uint4(0, 0, 0, 0);
    }
    if (t == 0) {
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
        tail->bar_ok = 1;
        fence_mbar_init();
        tma_prefetch_desc(&tmCB);
    }
    if (t < DM) tail->rowmax[t] = 0u;
    if (warp == 1) tmem_alloc(smem_addr(&tail->tmem_base), 32);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const BoundedWait wait{&tail->abort_flag, a.status, a.timeout_ns};

    // weight stream state (the producer lane starts only once X is quantized: weight requests
    // issued earlier would queue in front of X's loads and of the exchanges below)
    int stage = 0;
    uint32_t phase = 0, used = 0, last_parity = 0;
    int ptile = blockIdx.x, pit = 0;         // next (tile, k-block) to load
    auto produce = [&](int limit) -> bool {  // issue up to `limit` stage loads
        for (int n = 0; n < limit && ptile < a.tiles; ++n) {
            if (!wait(smem_addr(&tail->empty[stage]), phase ^ 1)) return false;
            const uint32_t full = smem_addr(&tail->full[stage]);
            mbar_arrive_expect_tx(full, DSTAGE);
            tma_load_2d(smem_addr(smem + stage * DSTAGE), &tmCB,
                        rotated_kblock(pit, ptile, a.kblocks) * DBK, ptile * DBM, full);
            used |= 1u << stage;
            last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
            if (++stage == S) {
                stage = 0;
                phase ^= 1;
            }
            if (++pit == a.kblocks) {
                pit = 0;
                ptile += gridDim.x;
            }
        }
        return true;
    };

    // ------------------------------------------------- quantize X across the grid ----
    // pass 1 (own columns): outlier bits (OR over the 16 lanes = rows of a chunk) to the
    // scratch, row maxima over the regular columns
    uint32_t fl[QKEEP];
    float rm = 0.0f;
#pragma unroll
    for (int i = 0; i < QKEEP; ++i) {
        fl[i] = 0;
        const int p = p0 + warp + i * DWARPS;
        if (p < p1) {                        // uniform over the warp
            float f[8];
            unpack8(keep[i], f);
            uint32_t b = outlier_bits(f, a.threshold);
#pragma unroll
            for (int o = 1; o < 16; o <<= 1) b |= __shfl_xor_sync(0xffffffffu, b, o);
            fl[i] = b;
            if (m == 0) a.scr->flags[2 * p + half] = (uint8_t)b;
            rm = masked_max(f, b, rm);
        }
    }
    for (int p = p0 + warp + QKEEP * DWARPS; p < p1; p += DWARPS) {
        const uint4 v = m < a.M ? __ldg(X4 + (int64_t)m * nchunks + 2 * p + half)
                                : make_uint4(0, 0, 0, 0);
        float f[8];
        unpack8(v, f);
        uint32_t b = outlier_bits(f, a.threshold);
#pragma unroll
        for (int o = 1; o < 16; o <<= 1) b |= __shfl_xor_sync(0xffffffffu, b, o);
        if (m == 0) a.scr->flags[2 * p + half] = (uint8_t)b;
        rm = masked_max(f, b, rm);
    }
    rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, 16));
    if (half == 0 && m < a.M && rm > 0.0f) atomicMax(&tail->rowmax[m], __float_as_uint(rm));
    __syncthreads();
    if (t < DM) a.scr->part[blockIdx.x * DM + t] = __uint_as_float(tail->rowmax[t]);
    grid_barrier(a.scr->arrived[0], a.epoch, tail, a.status);

    // every CTA: SCA (max over the CTAs' partial maxima), multipliers, ascending outlier list
    if (t < DM) tail->rowmax[t] = 0u;
    __syncthreads();
    {
        float r = 0.0f;
        for (int i = t; i < (int)gridDim.x * DM; i += DTHREADS)   // DTHREADS % DM == 0
            r = fmaxf(r, __ldcg(&a.scr->part[i]));
        // lanes l and l + 16 hold the same row
        r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, 16));
        if (half == 0 && r > 0.0f) atomicMax(&tail->rowmax[m], __float_as_uint(r));
    }
    {
        const int per = (nchunks + DTHREADS - 1) / DTHREADS;   // contiguous chunks per thread
        const int c0 = t * per, c1 = min(nchunks, c0 + per);
        uint32_t bits[(kDecodeMaxK / 8 + DTHREADS - 1) / DTHREADS];
        int cnt = 0;
#pragma unroll
        for (int j = 0; j < (int)(sizeof(bits) / sizeof(bits[0])); ++j) {
            bits[j] = (c0 + j < c1) ? (uint32_t)__ldcg(&a.scr->flags[c0 + j]) : 0u;
            cnt += __popc(bits[j]);
        }
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) tail->warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            const int v0 = lane < DWARPS ? tail->warp_tot[lane] : 0;
            int x = v0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane < DWARPS) tail->warp_tot[lane] = x - v0;
            if (lane == 31) {
                tail->n_out = min(x, a.cap);
                if (blockIdx.x == 0) {
                    *a.count = x;
                    a.status.set(x > a.cap ? LLMINT8_ERR_OUTLIER_CAPACITY : LLMINT8_OK);
                }
            }
        }
        __syncthreads();
        int pos = tail->warp_tot[warp] + incl - cnt;
#pragma unroll
        for (int j = 0; j < (int)(sizeof(bits) / sizeof(bits[0])); ++j) {
            uint32_t b = bits[j];
            while (b) {
                const int e = __ffs(b) - 1;
                b &= b - 1;
                if (pos < a.cap) tail->idx[pos] = (c0 + j) * 8 + e;
                ++pos;
            }
        }
    }
    if (t < DM) {
        const float amax = __uint_as_float(tail->rowmax[t]);
        tail->sca[t] = amax;
        tail->mult[t] = (t < a.M && amax > 0.0f) ? __fdiv_rn(127.0f, amax) : 0.0f;
    }
    __syncthreads();

    // pass 2 (own columns): int8 codes into the operand image, all 16 rows
    const float mul = tail->mult[m];
#pragma unroll
    for (int i = 0; i < QKEEP; ++i) {
        const int p = p0 + warp + i * DWARPS;
        if (p < p1) {
            const int c = 2 * p + half;
            uint2 q = make_uint2(0, 0);
            if (mul > 0.0f) {
                float f[8];
                unpack8(keep[i], f);
                q = quant8(f, mul, fl[i]);
            }
            *reinterpret_cast<uint2 *>(a.image + xq_offset(m, c * 8)) = q;
        }
    }
    for (int p = p0 + warp + QKEEP * DWARPS; p < p1; p += DWARPS) {
        const int c = 2 * p + half;
        uint2 q = make_uint2(0, 0);
        if (mul > 0.0f) {
            float f[8];
            unpack8(__ldg(X4 + (int64_t)m * nchunks + c), f);
            q = quant8(f, mul, (uint32_t)__ldcg(&a.scr->flags[c]));
        }
        *reinterpret_cast<uint2 *>(a.image + xq_offset(m, c * 8)) = q;
    }
    if (blockIdx.x == 0) {
        // the padding columns of the image
        const int kpad_chunks = a.kblocks * (DBK / 8);
        for (int i = t; i < (kpad_chunks - nchunks) * DM; i += DTHREADS)
            *reinterpret_cast<uint2 *>(a.image + xq_offset(i % DM, (nchunks + i / DM) * 8)) =
                make_uint2(0, 0);
    }
    // X at the outlier columns, [j][m]
    const int n_out = tail->n_out;
    for (int i = t; i < n_out * DM; i += DTHREADS) {
        const int j = i / DM, mm = i % DM;
        tail->xo[i] = mm < a.M ? a.X[(int64_t)mm * a.K + tail->idx[j]] : __float2half_rn(0.0f);
    }
    // the image is read by other SMs' bulk copies (async proxy)
    fence_proxy_async_global();
    grid_barrier(a.scr->arrived[1], a.epoch, tail, a.status);
    const bool run = tail->bar_ok != 0;

    if (warp == 0) {
        // --------------------------------------------------- weight stream (TMA) ----
        if (lane == 0) {
            if (run) produce(1 << 30);
            for (int s = 0; s < S; ++s)
                if (used & (1u << s))
                    drain_wait(smem_addr(&tail->full[s]), (last_parity >> s) & 1u, a.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issue ----
        if (lane == 0) {
            // the whole quantized X, written by every CTA of the grid
            const uint32_t xbar = smem_addr(&tail->xbar);
            const uint32_t img_bytes = (uint32_t)(a.kblocks * DBK * DM);
            fence_proxy_async_global();
            mbar_arrive_expect_tx(xbar, img_bytes);
            for (uint32_t off = 0; off < img_bytes; off += 16384)
                bulk_load_1d(smem_addr(xq) + off, a.image + off, min(16384u, img_bytes - off),
                             xbar);
            const bool have_x = run && wait(xbar, 0);
            const uint32_t idesc = idesc_i8(DBM, DM);
            const uint32_t xq_base = smem_addr(xq);
            int cs = 0, acc = 0;
            uint32_t cphase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; have_x && tile < a.tiles; tile += gridDim.x) {
                if (!wait(smem_addr(&tail->acc_empty[acc]), acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * DM);
                bool good = true;
                for (int it = 0; it < a.kblocks; ++it) {
                    const int kb = rotated_kblock(it, tile, a.kblocks);
                    if (!wait(smem_addr(&tail->full[cs]), cphase)) {
                        good = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + cs * DSTAGE);
                    const uint32_t sb = xq_base + (uint32_t)(kb * DM * 128);
#pragma unroll
                    for (int k = 0; k < DBK / 32; ++k)
                        mma_i8(d, sw128_desc(sa + 32 * k), sw128_desc(sb + 32 * k), idesc,
                               (it | k) != 0);
                    tc_commit(smem_addr(&tail->empty[cs]));
                    if (++cs == S) {
                        cs = 0;
                        cphase ^= 1;
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
    } else if (warp >= 4 && warp < 8) {
        // ------------------------------------------------------------------ epilogue ----
        const int qd = warp & 3;
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        const float inv = 1.0f / 16129.0f;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; run && tile < a.tiles; tile += gridDim.x) {
            int okw = 0;
            if (lane == 0) okw = wait(smem_addr(&tail->acc_full[acc]), acc_phase) ? 1 : 0;
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!okw) break;
            tc_fence_after();
            uint32_t d[DM];
            tmem_ld_32x16(tl + (uint32_t)(acc * DM), d);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&tail->acc_empty[acc]));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;

            const int n = tile * DBM + qd * 32 + lane;
            if (n < a.N) {
                const float sb = a.SCB[n];
                const float b = a.bias ? __half2float(a.bias[n]) : 0.0f;
                float o[DM];
#pragma unroll
                for (int r = 0; r < DM; ++r) o[r] = 0.0f;
                const int8_t *cbrow = a.CB + (int64_t)n * a.K;
                for (int j = 0; j < n_out; ++j) {
                    const int col = tail->idx[j];
                    const float w = a.W16 ? __half2float(a.W16[(int64_t)n * a.K + col])
                                          : __half2float(__float2half_rn(__fdiv_rn(
                                                __fmul_rn((float)cbrow[col], sb), 127.0f)));
                    const uint4 *xv = reinterpret_cast<const uint4 *>(tail->xo + j * DM);
                    float f0[8], f1[8];
                    unpack8(xv[0], f0);
                    unpack8(xv[1], f1);
#pragma unroll
                    for (int r = 0; r < 8; ++r) {
                        o[r] = fmaf(f0[r], w, o[r]);
                        o[r + 8] = fmaf(f1[r], w, o[r + 8]);
                    }
                }
#pragma unroll
                for (int r = 0; r < DM; ++r) {
                    if (r < a.M) {
                        const float y = fmaf((float)(int32_t)d[r], tail->sca[r] * inv * sb,
                                             o[r] + b);
                        a.Y[(int64_t)r * a.N + n] = __float2half_rn(y);
                        if (a.C_debug) a.C_debug[(int64_t)r * a.N + n] = (int32_t)d[r];
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 32);
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

    DArgs a;
    a.X = d.X;
    a.CB = d.CB;
    a.SCB = d.SCB;
    a.W16 = d.W16;
    a.bias = d.bias;
    a.Y = d.Y;
    a.C_debug = d.C_debug;
    a.count = d.count;
    a.scr = d.scratch;
    a.image = reinterpret_cast<uint8_t *>(d.scratch) + sizeof(DecodeScratch);
    a.status = d.status;
    a.epoch = d.status.tag >> 4;
    a.M = (int)d.M;
    a.N = (int)d.N;
    a.K = (int)d.K;
    a.cap = (int)d.cap;
    a.threshold = d.threshold;
    a.kblocks = (int)ceil_div(d.K, DBK);
    a.tiles = (int)ceil_div(d.N, DBM);
    a.timeout_ns = d.timeout_ns;
    // shared memory: [stages][quantized X][tail], 1024-byte aligned pieces
    const int xq_bytes = a.kblocks * DBK * DM;
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

    // every CTA must be resident at once (they meet at grid barriers): cooperative launch,
    // one CTA per SM (the shared memory allows no more)
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.gridDim = dim3((unsigned)std::min({a.tiles, sms, kDecodeMaxGrid}));
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

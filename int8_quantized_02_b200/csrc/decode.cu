// Decode path of the LLM.int8() layer (few activation rows, M <= 16).
//
// At decode sizes the layer is bound by streaming the int8 weight CB from HBM once, and the
// rest must hide under that stream.  One kernel in clusters of 4 CTAs (512 threads, one CTA
// per SM, one 128-row weight tile per CTA, grid-stride when there are more tiles):
//
//   warps 1..15   quantize X, each CTA of the cluster 1/4 of the columns: one lane per (row,
//                 8-column chunk), each warp holding all 16 rows of two chunks, values in
//                 registers.  The outlier bits of a chunk (|x| >= threshold in any row) are an
//                 OR across its 16 lanes; the row maxima over the regular columns reduce in
//                 registers and across warps.  Bits and partial maxima go to every CTA of the
//                 cluster through distributed shared memory; after a cluster barrier each CTA
//                 has SCA and the ascending outlier set, quantizes its columns and writes the
//                 int8 codes straight into every CTA's operand buffer (128-byte swizzled
//                 K-major, rows padded to 16, outlier columns 0), with X at its outlier
//                 columns into their outlier tables; a second cluster barrier and every CTA
//                 holds the whole quantized X.  Nothing of this goes through L2 or HBM but
//                 the first load of X;
//   warp 0        TMA producer: once its CTA's X loads have landed (weight requests issued
//                 earlier would queue in front of them) it fills a ring of shared-memory
//                 stages with 128-row x 128-byte tiles of CB (16 KB) - that needs nothing
//                 from X - and keeps streaming after the barriers;
//   warp 1        tcgen05.mma kind::i8 with the weight tile as the 128-row operand and the
//                 quantized X as the 16-column operand: D[n, m] = sum_k CB[n, k] Xq[m, k] into
//                 a 128 x 16 int32 TMEM accumulator (double-buffered over tiles);
//   warps 4..7    epilogue: D -> registers; y = D * SCA_m * SCB_n / 127^2
//                 + sum_{j in O} X[m, O_j] * W_o[n, O_j] + bias_n (the fp16 outlier part of
//                 the decomposition, weights from the bytes of the outlier columns) -> fp16.
// Same method and rounding as the GEMM path (LLM.int8() summary, sections الابتكار الثاني
// and الصورة الكاملة; blog sections MatMul 内部 and 用法).  Every wait is bounded; every
// thread of every CTA reaches each cluster barrier exactly once, with no wait in between
// that depends on another CTA.
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
constexpr int QWARPS = DWARPS - 1;      // warps 1..15 quantize X
constexpr int QTHREADS = QWARPS * 32;
constexpr int DMAX_STAGES = 12;
constexpr int DCAP = kDecodeMaxOutliers;
constexpr int CL = 4;                   // CTAs per cluster
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in per CTA
// chunk pairs per quantization warp: every pair of this CTA's columns stays in registers
constexpr int QKEEP = (kDecodeMaxK / 16 / CL + QWARPS - 1) / QWARPS;

struct DTail {
    uint64_t full[DMAX_STAGES];
    uint64_t empty[DMAX_STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint64_t xin;                        // this CTA's X loads have landed
    uint32_t tmem_base;
    int abort_flag;
    int n_out;                           // outlier columns used (<= cap)
    int pad0;
    uint32_t pmax[DM];                   // this CTA's row maxima (float bits, >= 0)
    float part[CL][DM];                  // row maxima of every CTA of the cluster
    float sca[DM];
    float mult[DM];                      // fl32(127 / sca), 0 for rows >= M or all-zero rows
    int warp_tot[DWARPS];
    alignas(16) uint8_t flags[kDecodeMaxK / 8];   // outlier bits of every 8-column chunk
    int32_t idx[DCAP];                   // outlier columns (ascending)
    alignas(16) __half xo[DCAP * DM];    // X at the outlier columns, [j][m] (read as uint4)
};
static_assert(offsetof(DTail, xo) % 16 == 0, "xo is read with 16-byte loads");
static_assert(offsetof(DTail, xin) % 8 == 0, "mbarriers are 8-byte aligned");

struct DArgs {
    const __half *X;
    const int8_t *CB;
    const float *SCB;
    const __half *W16;
    const __half *bias;
    __half *Y;
    int32_t *C_debug;
    int32_t *count;
    StatusRef status;
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

__device__ __forceinline__ void st_cluster_v2(uint32_t addr, const uint2 &v) {
    asm volatile("st.shared::cluster.v2.u32 [%0], {%1, %2};" ::"r"(addr), "r"(v.x), "r"(v.y)
                 : "memory");
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
    const uint32_t rank = cluster_ctarank();
    const int m = lane & 15;                 // quantization: the row this lane handles
    const int half = lane >> 4;              //               which chunk of the warp's pair
    const int qw = warp - 1;                 // quantization warp index (warps 1..15)
    const int nchunks = a.K / 8;
    const int npairs = nchunks / 2;          // K is a multiple of 16
    const int pp = (npairs + CL - 1) / CL;
    const int p0 = (int)rank * pp, p1 = min(npairs, p0 + pp);   // this CTA's pairs
    const uint4 *X4 = reinterpret_cast<const uint4 *>(a.X);

    // this CTA's columns of X, first of all memory traffic
    uint4 keep[QKEEP];
#pragma unroll
    for (int i = 0; i < QKEEP; ++i) {
        const int p = p0 + qw + i * QWARPS;
        keep[i] = (warp > 0 && p < p1 && m < a.M)
                      ? __ldg(X4 + (int64_t)m * nchunks + 2 * p + half)
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
        mbar_init(smem_addr(&tail->xin), 1);
        tail->abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmCB);
    }
    if (t < DM) tail->pmax[t] = 0u;
    if (warp == 1) tmem_alloc(smem_addr(&tail->tmem_base), 32);
    // zero the operand (rows >= M and columns >= K must read as 0)
    for (int i = t; i < a.kblocks * DBK * DM / 16; i += DTHREADS)
        reinterpret_cast<uint4 *>(xq)[i] = make_uint4(0, 0, 0, 0);
    tc_fence_before();
    // every CTA's barriers and zeroed buffers exist before a peer writes into them
    cluster_barrier_all();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const BoundedWait wait{&tail->abort_flag, a.status, a.timeout_ns};

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

    uint32_t fl[QKEEP];
    if (warp == 0) {
        // the ring fill needs no free slot (they all start empty) and nothing from X; it
        // waits for this CTA's X loads so as not to queue in front of them
        if (lane == 0) {
            drain_wait(smem_addr(&tail->xin), 0, a.status);
            produce(S);
        }
        __syncwarp();
    } else {
        // ------------------------------- quantize X, this CTA's quarter of the columns ----
        float rm = 0.0f;
#pragma unroll
        for (int i = 0; i < QKEEP; ++i) {
            fl[i] = 0;
            const int p = p0 + qw + i * QWARPS;
            if (p < p1) {                    // uniform over the warp
                float f[8];
                unpack8(keep[i], f);
                uint32_t b = outlier_bits(f, a.threshold);
#pragma unroll
                for (int o = 1; o < 16; o <<= 1) b |= __shfl_xor_sync(0xffffffffu, b, o);
                fl[i] = b;
                if (m == 0) {
                    const uint32_t dst = smem_addr(&tail->flags[2 * p + half]);
                    for (int r = 0; r < CL; ++r) st_cluster_u8(map_to_rank(dst, (uint32_t)r), b);
                }
                rm = masked_max(f, b, rm);
            }
        }
        rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, 16));
        if (half == 0 && m < a.M && rm > 0.0f) atomicMax(&tail->pmax[m], __float_as_uint(rm));
        named_barrier(1, QTHREADS);
        if (t == 32) mbar_arrive(smem_addr(&tail->xin));   // X is in: the ring may fill
        if (t >= 32 && t < 32 + DM) {
            const int q = t - 32;
            const uint32_t dst = smem_addr(&tail->part[rank][q]);
            for (int r = 0; r < CL; ++r)
                st_cluster_u32(map_to_rank(dst, (uint32_t)r), tail->pmax[q]);
        }
    }
    // ---------------------------------- exchange 1: outlier bits and row maxima ----
    __syncwarp();
    cluster_barrier_all();

    if (warp > 0) {
        const int q = t - 32;                // 0 .. QTHREADS-1
        if (q < DM) {
            float amax = 0.0f;
            for (int r = 0; r < CL; ++r) amax = fmaxf(amax, tail->part[r][q]);
            tail->sca[q] = amax;
            tail->mult[q] = (q < a.M && amax > 0.0f) ? __fdiv_rn(127.0f, amax) : 0.0f;
        }
        // ascending outlier list: contiguous chunks per thread, scan over warps 1..15
        const int per = (nchunks + QTHREADS - 1) / QTHREADS;
        const int c0 = q * per, c1 = min(nchunks, c0 + per);
        int cnt = 0;
        for (int c = c0; c < c1; ++c) cnt += __popc(tail->flags[c]);
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) tail->warp_tot[qw] = incl;
        named_barrier(1, QTHREADS);
        if (qw == 0) {
            const int v0 = lane < QWARPS ? tail->warp_tot[lane] : 0;
            int x = v0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (lane < QWARPS) tail->warp_tot[lane] = x - v0;
            if (lane == 31) {
                tail->n_out = min(x, a.cap);
                if (blockIdx.x == 0) {
                    *a.count = x;
                    a.status.set(x > a.cap ? LLMINT8_ERR_OUTLIER_CAPACITY : LLMINT8_OK);
                }
            }
        }
        named_barrier(1, QTHREADS);
        int pos = tail->warp_tot[qw] + incl - cnt;
        for (int c = c0; c < c1; ++c) {
            uint32_t b = tail->flags[c];
            while (b) {
                const int e = __ffs(b) - 1;
                b &= b - 1;
                if (pos < a.cap) tail->idx[pos] = c * 8 + e;
                ++pos;
            }
        }
        named_barrier(1, QTHREADS);

        // int8 codes of this CTA's columns into every CTA's operand; X at outlier columns
        const float mul = tail->mult[m];
        const int n_out = tail->n_out;
        const uint32_t xq_base = smem_addr(xq);
        const uint32_t xo_base = smem_addr(tail->xo);
#pragma unroll
        for (int i = 0; i < QKEEP; ++i) {
            const int p = p0 + qw + i * QWARPS;
            if (p < p1) {
                const int c = 2 * p + half;
                float f[8];
                unpack8(keep[i], f);
                if (mul > 0.0f) {
                    const uint2 qv = quant8(f, mul, fl[i]);
                    const uint32_t dst = xq_base + xq_offset(m, c * 8);
                    for (int r = 0; r < CL; ++r) st_cluster_v2(map_to_rank(dst, (uint32_t)r), qv);
                }
                if (fl[i]) {
                    // this chunk holds outlier columns: find their list positions
                    for (int j = 0; j < n_out; ++j) {
                        const int col = tail->idx[j];
                        if ((col >> 3) == c) {
                            const __half hv = __float2half_rn(m < a.M ? f[col & 7] : 0.0f);
                            const uint32_t dst = xo_base + 2u * (uint32_t)(j * DM + m);
                            for (int r = 0; r < CL; ++r)
                                st_cluster_u16(map_to_rank(dst, (uint32_t)r),
                                               __half_as_ushort(hv));
                        }
                    }
                }
            }
        }
    }
    // ------------------------------------------- exchange 2: the quantized operand ----
    __syncwarp();
    cluster_barrier_all();
    const int n_out = tail->n_out;

    if (warp == 0) {
        // --------------------------------------------------- weight stream (TMA) ----
        if (lane == 0) {
            produce(1 << 30);
            for (int s = 0; s < S; ++s)
                if (used & (1u << s))
                    drain_wait(smem_addr(&tail->full[s]), (last_parity >> s) & 1u, a.status);
        }
    } else if (warp == 1) {
        // ------------------------------------------------------------- MMA issue ----
        if (lane == 0) {
            // peers wrote the operand through the generic proxy; the tensor core reads it
            // through the async proxy
            fence_proxy_async_smem();
            const uint32_t idesc = idesc_i8(DBM, DM);
            const uint32_t xq_base = smem_addr(xq);
            int cs = 0, acc = 0;
            uint32_t cphase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
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
        for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
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
    static int max_clusters[64] = {0};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;

    DArgs a;
    a.X = d.X;
    a.CB = d.CB;
    a.SCB = d.SCB;
    a.W16 = d.W16;
    a.bias = d.bias;
    a.Y = d.Y;
    a.C_debug = d.C_debug;
    a.count = d.count;
    a.status = d.status;
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

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(DTHREADS);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int clusters;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (max_clusters[dev] == 0) {
            err = cudaFuncSetAttribute(llmint8_decode_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_LIMIT);
            if (err != cudaSuccess) return err;
            cudaLaunchConfig_t qc = cfg;
            qc.gridDim = dim3(CL);
            qc.dynamicSmemBytes = (size_t)SMEM_LIMIT;
            int n = 0;
            err = cudaOccupancyMaxActiveClusters(&n, llmint8_decode_kernel, &qc);
            if (err != cudaSuccess) return err;
            if (n < 1) return cudaErrorInvalidConfiguration;
            max_clusters[dev] = n;
        }
        clusters = max_clusters[dev];
    }
    clusters = std::min<int>(clusters, (int)ceil_div(a.tiles, CL));
    cfg.gridDim = dim3((unsigned)(clusters * CL));

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
    err = cudaLaunchKernelEx(&cfg, llmint8_decode_kernel, tm, a);
    note_launches(1);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace llmint8

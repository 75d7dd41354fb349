// Single-launch decode path of the LLM.int8() layer (few activation rows, M <= 16).
//
// At decode sizes the layer is bound by streaming the int8 weight CB from HBM once.  The
// kernel runs in clusters of 8 CTAs (one CTA per SM) and never lets the weight stream wait
// on more than the first few stages:
//   warp 0        TMA producer: streams 128-row x 128-byte tiles of CB (16 KB) through a
//                 ring of shared-memory stages, from the moment its CTA's slice of X landed;
//   warps 1..7    quantize X cooperatively inside the cluster.  CTA r of the cluster owns
//                 1/8 of the columns: it bulk-copies those columns of every row, finds which
//                 are outlier columns (|x| >= threshold in any row) and the row maxima over
//                 its regular columns, and publishes both to every CTA of the cluster through
//                 distributed shared memory.  After a cluster exchange each CTA has the full
//                 outlier set and SCA (max over the 8 partial maxima); CTA r then quantizes
//                 its columns and writes the int8 bytes straight into the 128-byte-swizzled
//                 K-major operand buffer of every CTA of the cluster (and the fp16 values of
//                 its outlier columns into their outlier tables).  After a second exchange
//                 every CTA holds the whole quantized X (rows padded to 16, outlier columns 0);
//   warp 1        issues tcgen05.mma kind::i8 with the weight tile as the 128-row operand and
//                 the quantized X as the 16-column operand: D[n, m] = sum_k CB[n, k] Xq[m, k]
//                 into a 128 x 16 int32 TMEM accumulator (double-buffered over tiles);
//   warps 4..7    epilogue: D -> registers; y = D * SCA_m * SCB_n / 127^2
//                 + sum_{j in O} X[m, O_j] * W_o[n, O_j] + bias_n (the fp16 outlier part of
//                 the decomposition, from the weight bytes of the outlier columns) -> fp16.
// Same method and rounding as the GEMM path (LLM.int8() summary, sections الابتكار الثاني
// and الصورة الكاملة; blog sections MatMul 内部 and 用法), with the work laid out for a
// weight-bandwidth-bound shape.  Pipeline waits are bounded (BoundedWait); the waits of the
// cluster exchange use the fixed drain bound, so every CTA always reaches both exchanges.
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
constexpr int QTHREADS = DTHREADS - 32; // warps 1..7 quantize X
constexpr int DMAX_STAGES = 12;
constexpr int DCAP = kDecodeMaxOutliers;
constexpr int CL = 8;                   // CTAs per cluster
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in per CTA
// Columns owned by one CTA of the cluster: a multiple of 32 (one flag word = 4 chunks of 8).
constexpr int kMaxOwnCols = ((kDecodeMaxK / CL + 31) / 32) * 32;

struct DTail {
    uint64_t full[DMAX_STAGES];
    uint64_t empty[DMAX_STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint64_t xbar;                       // this CTA's slice of X has landed
    uint64_t cbar;                       // cluster exchange: one arrival per CTA of the cluster
    uint32_t tmem_base;
    int abort_flag;
    int n_out;                           // outlier columns used (<= cap)
    int n_total;                         // outlier columns found
    uint32_t pmax[DM];                   // this CTA's row maxima (float bits, >= 0)
    float part[CL][DM];                  // row maxima of every CTA of the cluster
    float sca[DM];
    float mult[DM];                      // fl32(127 / sca), 0 for an all-zero row
    uint8_t myflags[kMaxOwnCols / 8];    // outlier bits of this CTA's chunks
    alignas(16) uint8_t flags[kDecodeMaxK / 8];   // outlier bits of every 8-column chunk
    int32_t idx[DCAP];                   // outlier columns (ascending)
    alignas(16) __half xo[DCAP * DM];    // X at the outlier columns, [j][m] (read as uint4)
};

static_assert(offsetof(DTail, xo) % 16 == 0, "xo is read with 16-byte loads");
static_assert(offsetof(DTail, flags) % 4 == 0, "flags are written as 32-bit words");
static_assert(offsetof(DTail, full) % 8 == 0 && offsetof(DTail, xbar) % 8 == 0 &&
                  offsetof(DTail, cbar) % 8 == 0,
              "mbarriers are 8-byte aligned");

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
    int own_cols;                        // columns per CTA of the cluster (multiple of 32)
    uint32_t xq_off;                     // byte offsets in shared memory
    uint32_t stash_off;
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

// Four absmax-quantized int8 codes packed little-endian; a set bit in `skip` gives 0.
__device__ __forceinline__ uint32_t quant4(const float *f, float mul, uint32_t skip) {
    uint32_t w = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        int q = 0;
        if (!((skip >> e) & 1u)) q = max(-127, min(127, __float2int_rn(__fmul_rn(f[e], mul))));
        w |= (uint32_t)(q & 0xff) << (8 * e);
    }
    return w;
}

// Exchange point of the quantization warps of every CTA of the cluster: the shared-memory
// writes made before it (locally or into peers) are visible to every CTA after it.
__device__ __forceinline__ bool cluster_exchange(DTail *tail, uint32_t parity, StatusRef status) {
    fence_acq_rel_cluster();
    named_barrier(1, QTHREADS);
    if (threadIdx.x == 32) {
        const uint32_t bar = smem_addr(&tail->cbar);
        for (int r = 0; r < CL; ++r) mbar_arrive_cluster(map_to_rank(bar, (uint32_t)r));
        constexpr uint64_t kLimitNs = 1000000000ull;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t it = 0;; ++it) {
            if (mbar_try_wait_cluster(bar, parity)) break;
            if ((it & 63u) == 0u && global_timer_ns() - t0 > kLimitNs) {
                status.timed_out();
                tail->abort_flag = 1;
                break;
            }
        }
    }
    named_barrier(1, QTHREADS);
    return !tail->abort_flag;
}

__global__ void __launch_bounds__(DTHREADS, 1)
llmint8_decode_kernel(const __grid_constant__ CUtensorMap tmCB, const DArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DTail *tail = reinterpret_cast<DTail *>(smem + a.tail_off);
    uint8_t *xq = smem + a.xq_off;
    __half *stash = reinterpret_cast<__half *>(smem + a.stash_off);   // [m][own_cols]
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = threadIdx.x;
    const int S = a.stages;
    const uint32_t rank = cluster_ctarank();
    // this CTA's columns [col0, col0 + ncols)
    const int col0 = (int)rank * a.own_cols;
    const int ncols = max(0, min(a.own_cols, a.K - col0));

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
        mbar_init(smem_addr(&tail->cbar), CL);
        tail->abort_flag = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmCB);
    }
    if (t < DM) tail->pmax[t] = 0u;
    if (warp == 1) tmem_alloc(smem_addr(&tail->tmem_base), 32);
    // zero the operand: rows >= M, columns >= K and all-zero rows must read as 0
    for (int i = t; i < a.kblocks * DBK * DM / 16; i += DTHREADS)
        reinterpret_cast<uint4 *>(xq)[i] = make_uint4(0, 0, 0, 0);
    tc_fence_before();
    // every CTA's mbarriers and zeroed operand exist before any peer may touch them
    cluster_barrier_all();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const BoundedWait wait{&tail->abort_flag, a.status, a.timeout_ns};

    if (t == 0) {
        // this CTA's columns of every row of X
        const uint32_t bar = smem_addr(&tail->xbar);
        mbar_arrive_expect_tx(bar, (uint32_t)(a.M * ncols * 2));
        if (ncols > 0)
            for (int m = 0; m < a.M; ++m)
                bulk_load_1d(smem_addr(stash + m * a.own_cols), a.X + (int64_t)m * a.K + col0,
                             (uint32_t)(ncols * 2), bar);
    }

    if (warp == 0) {
        // --------------------------------------------------- weight stream (TMA) ----
        if (lane == 0) {
            // start once this CTA's X slice is in: started earlier, that copy would queue
            // behind the weight requests of every SM
            const bool go = drain_wait(smem_addr(&tail->xbar), 0, a.status);
            int stage = 0;
            uint32_t phase = 0, used = 0, last_parity = 0;
            for (int tile = blockIdx.x; go && tile < a.tiles; tile += gridDim.x) {
                const int n0 = tile * DBM;
                for (int it = 0; it < a.kblocks; ++it) {
                    const int kb = rotated_kblock(it, tile, a.kblocks);
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
    } else {
        // --------------------------- cooperative quantization of X (warps 1..7) ----
        const int q = t - 32;                            // 0 .. QTHREADS-1
        const int nchunk = ncols / 8;
        const bool have_x = drain_wait(smem_addr(&tail->xbar), 0, a.status);
        // outlier bits of this CTA's 8-column chunks (every row counts)
        for (int c = q; c < nchunk; c += QTHREADS) {
            uint32_t fl = 0;
            for (int m = 0; have_x && m < a.M; ++m) {
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(stash + m * a.own_cols + c * 8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) fl |= (fabsf(f[e]) >= a.threshold ? 1u : 0u) << e;
            }
            tail->myflags[c] = (uint8_t)fl;
        }
        named_barrier(1, QTHREADS);
        // publish them as 32-bit words to every CTA; row maxima over the regular columns
        const uint32_t flags_base = smem_addr(tail->flags) + (uint32_t)(col0 / 8);
        for (int w = q; w < (nchunk + 3) / 4; w += QTHREADS) {
            uint32_t word = 0;
            for (int b = 0; b < 4 && 4 * w + b < nchunk; ++b)
                word |= (uint32_t)tail->myflags[4 * w + b] << (8 * b);
            for (int r = 0; r < CL; ++r)
                st_cluster_u32(map_to_rank(flags_base + 4u * w, (uint32_t)r), word);
        }
        for (int m = 0; have_x && m < a.M; ++m) {
            float r = 0.0f;
            for (int c = q; c < nchunk; c += QTHREADS) {
                const uint32_t fl = tail->myflags[c];
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(stash + m * a.own_cols + c * 8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (!((fl >> e) & 1u)) r = fmaxf(r, fabsf(f[e]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, o));
            if (lane == 0 && r > 0.0f) atomicMax(&tail->pmax[m], __float_as_uint(r));
        }
        named_barrier(1, QTHREADS);
        if (q < DM) {
            const uint32_t dst = smem_addr(&tail->part[rank][q]);
            const uint32_t v = q < a.M ? tail->pmax[q] : 0u;
            for (int r = 0; r < CL; ++r) st_cluster_u32(map_to_rank(dst, (uint32_t)r), v);
        }
        cluster_exchange(tail, 0, a.status);

        // every CTA now has all flags and partial maxima: SCA, multipliers, outlier list
        if (q < DM) {
            float amax = 0.0f;
            for (int r = 0; r < CL; ++r) amax = fmaxf(amax, tail->part[r][q]);
            tail->sca[q] = amax;
            tail->mult[q] = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
        }
        if (warp == 1) {
            const int nch_all = a.K / 8;
            const int per = (nch_all + 31) / 32;
            const int c0 = lane * per, c1 = min(nch_all, c0 + per);
            int cnt = 0;
            for (int c = c0; c < c1; ++c) cnt += __popc(tail->flags[c]);
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += y;
            }
            int pos = incl - cnt;
            for (int c = c0; c < c1; ++c) {
                uint32_t fl = tail->flags[c];
                while (fl) {
                    const int e = __ffs(fl) - 1;
                    fl &= fl - 1;
                    if (pos < a.cap) tail->idx[pos] = c * 8 + e;
                    ++pos;
                }
            }
            const int total = __shfl_sync(0xffffffffu, incl, 31);
            if (lane == 0) {
                tail->n_total = total;
                tail->n_out = min(total, a.cap);
                if (blockIdx.x == 0) {
                    *a.count = total;
                    a.status.set(total > a.cap ? LLMINT8_ERR_OUTLIER_CAPACITY : LLMINT8_OK);
                }
            }
        }
        named_barrier(1, QTHREADS);

        // quantize this CTA's columns, 16 at a time, into every CTA's operand buffer
        const int ngroups = ncols / 16;
        const uint32_t xq_base = smem_addr(xq);
        for (int i = q; have_x && i < a.M * ngroups; i += QTHREADS) {
            const int m = i / ngroups, g = i - m * ngroups;
            const float mul = tail->mult[m];
            if (mul > 0.0f) {
                const uint32_t fl =
                    tail->myflags[2 * g] | ((uint32_t)tail->myflags[2 * g + 1] << 8);
                const uint4 *src =
                    reinterpret_cast<const uint4 *>(stash + m * a.own_cols + g * 16);
                float f[16];
                unpack8(src[0], f);
                unpack8(src[1], f + 8);
                uint4 v;
                v.x = quant4(f, mul, fl);
                v.y = quant4(f + 4, mul, fl >> 4);
                v.z = quant4(f + 8, mul, fl >> 8);
                v.w = quant4(f + 12, mul, fl >> 12);
                const uint32_t dst = xq_base + xq_offset(m, col0 + g * 16);
                for (int r = 0; r < CL; ++r) st_cluster_v4(map_to_rank(dst, (uint32_t)r), v);
            }
        }
        // the fp16 values of this CTA's outlier columns, [j][m], into every CTA
        {
            const int n_out = tail->n_out;
            const uint32_t xo_base = smem_addr(tail->xo);
            for (int i = q; have_x && i < n_out * DM; i += QTHREADS) {
                const int j = i / DM, m = i % DM;
                const int col = tail->idx[j];
                if (col >= col0 && col < col0 + ncols) {
                    const __half v = m < a.M ? stash[m * a.own_cols + (col - col0)]
                                             : __float2half_rn(0.0f);
                    const uint16_t bits = __half_as_ushort(v);
                    for (int r = 0; r < CL; ++r)
                        st_cluster_u16(map_to_rank(xo_base + 2u * i, (uint32_t)r), bits);
                }
            }
        }
        cluster_exchange(tail, 1, a.status);
        // the operand was written through the generic proxy; the tensor core reads it
        // through the async proxy
        fence_proxy_async_smem();
        named_barrier(1, QTHREADS);
        const bool run = have_x && !tail->abort_flag;
        const int n_out = tail->n_out;

        if (warp == 1) {
            // ------------------------------------------------------------- MMA issue ----
            if (lane == 0) {
                const uint32_t idesc = idesc_i8(DBM, DM);
                int stage = 0, acc = 0;
                uint32_t phase = 0, acc_phase = 0;
                for (int tile = blockIdx.x; run && tile < a.tiles; tile += gridDim.x) {
                    if (!wait(smem_addr(&tail->acc_empty[acc]), acc_phase ^ 1)) break;
                    tc_fence_after();
                    const uint32_t d = tmem + (uint32_t)(acc * DM);
                    bool good = true;
                    for (int it = 0; it < a.kblocks; ++it) {
                        const int kb = rotated_kblock(it, tile, a.kblocks);
                        if (!wait(smem_addr(&tail->full[stage]), phase)) {
                            good = false;
                            break;
                        }
                        tc_fence_after();
                        const uint32_t sa = smem_addr(smem + stage * DSTAGE);
                        const uint32_t sb = xq_base + (uint32_t)(kb * DM * 128);
#pragma unroll
                        for (int k = 0; k < DBK / 32; ++k)
                            mma_i8(d, sw128_desc(sa + 32 * k), sw128_desc(sb + 32 * k), idesc,
                                   (it | k) != 0);
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
                tc_commit(smem_addr(&tail->mma_done));
                drain_wait(smem_addr(&tail->mma_done), 0, a.status);
            }
        } else if (warp >= 4) {
            // -------------------------------------------------------------- epilogue ----
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
                    for (int m = 0; m < DM; ++m) o[m] = 0.0f;
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
                        for (int m = 0; m < 8; ++m) {
                            o[m] = fmaf(f0[m], w, o[m]);
                            o[m + 8] = fmaf(f1[m], w, o[m + 8]);
                        }
                    }
#pragma unroll
                    for (int m = 0; m < DM; ++m) {
                        if (m < a.M) {
                            const float y = fmaf((float)(int32_t)d[m], tail->sca[m] * inv * sb,
                                                 o[m] + b);
                            a.Y[(int64_t)m * a.N + n] = __float2half_rn(y);
                            if (a.C_debug) a.C_debug[(int64_t)m * a.N + n] = (int32_t)d[m];
                        }
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

// Shared memory: [stages][quantized X operand][X slice][tail], 1024-byte aligned pieces.
struct Shape {
    int stages = 0, smem = 0;
    uint32_t xq_off = 0, stash_off = 0, tail_off = 0;
};

Shape plan_smem(int kblocks, int own_cols) {
    Shape sh;
    const int xq_bytes = kblocks * DBK * DM;
    const int stash_bytes = (int)align_up(DM * own_cols * 2, 1024);
    const int tail_bytes = (int)align_up(sizeof(DTail), 1024);
    const int room = SMEM_LIMIT - 1024 - xq_bytes - stash_bytes - tail_bytes;
    sh.stages = std::min(DMAX_STAGES, room / DSTAGE);
    sh.xq_off = (uint32_t)(sh.stages * DSTAGE);
    sh.stash_off = sh.xq_off + (uint32_t)xq_bytes;
    sh.tail_off = sh.stash_off + (uint32_t)stash_bytes;
    sh.smem = (int)(sh.tail_off + sizeof(DTail) + 1024);
    return sh;
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
    a.own_cols = (int)align_up(ceil_div(d.K, CL), 32);
    a.timeout_ns = d.timeout_ns;
    // every plan fits in SMEM_LIMIT, which sizes the attribute and the occupancy query once
    const Shape worst = plan_smem(kDecodeMaxK / DBK, kMaxOwnCols);
    const Shape sh = plan_smem(a.kblocks, a.own_cols);
    if (worst.stages < 2 || sh.stages < 2 || a.own_cols > kMaxOwnCols || sh.smem > SMEM_LIMIT)
        return cudaErrorInvalidValue;
    a.stages = sh.stages;
    a.xq_off = sh.xq_off;
    a.stash_off = sh.stash_off;
    a.tail_off = sh.tail_off;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.blockDim = dim3(DTHREADS);
    cfg.dynamicSmemBytes = (size_t)sh.smem;
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

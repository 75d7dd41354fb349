// Single-launch decode path of the LLM.int8() layer (few activation rows, M <= 16).
//
// At decode sizes the layer is bound by streaming the int8 weight CB from HBM once, so the
// whole method runs in one kernel that never stops the weight stream:
//   all warps     first quantize X for this CTA (every CTA redundantly; X is a few hundred
//                 KB at most and stays in L2): per 8-column chunk one thread sees all rows,
//                 so it knows which of its columns are outliers (|x| >= threshold in any row)
//                 and the row maxima over its regular columns; block-wide maxima give SCA;
//                 the int8 rows are written straight into shared memory in the
//                 128-byte-swizzled K-major layout the tensor core reads, outlier columns 0.
//                 This runs before the weight stream starts: started together, the X loads
//                 queue behind every SM's weight requests and take several times longer;
//   warp 0        TMA producer: streams 128-row x 128-byte tiles of CB (16 KB) through a
//                 ring of shared-memory stages;
//   warp 1        issues tcgen05.mma kind::i8 with the weight tile as the 128-row
//                 operand and the quantized X (padded to 16 rows) as the 16-column operand:
//                 D[n, m] = sum_k CB[n, k] * Xq[m, k] into a 128 x 16 int32 TMEM
//                 accumulator (double-buffered over tiles);
//   warps 4..7    epilogue: D -> registers; y = D * SCA_m * SCB_n / 127^2
//                 + sum_{j in O} X[m, O_j] * W_o[n, O_j] + bias_n (the fp16 outlier part of
//                 the decomposition, from the weight bytes of the outlier columns) -> fp16.
// Same method and rounding as the GEMM path (LLM.int8() summary, sections الابتكار الثاني
// and الصورة الكاملة; blog sections MatMul 内部 and 用法), only the work is laid out for a
// weight-bandwidth-bound shape.  Every wait is bounded (BoundedWait).
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
constexpr int DCAP = kDecodeMaxOutliers;
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in per CTA

struct DTail {
    uint64_t full[DMAX_STAGES];
    uint64_t empty[DMAX_STAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint32_t tmem_base;
    int abort_flag;
    int n_out;                           // outlier columns used (<= cap)
    int n_total;                         // outlier columns found
    uint32_t rowmax[DM];                 // float bits (non-negative: int order == float order)
    float sca[DM];
    float mult[DM];                      // fl32(127 / sca), 0 for an all-zero row
    uint64_t xbar;                       // completion of the bulk copies of X
    uint8_t flags[kDecodeMaxK / 8];      // per 8-column chunk: outlier bit per column
    int32_t idx[DCAP];                   // outlier columns (ascending)
    alignas(16) __half xo[DCAP * DM];    // X at the outlier columns, [j][m] (read as uint4)
};

static_assert(offsetof(DTail, xo) % 16 == 0, "xo is read with 16-byte loads");
static_assert(offsetof(DTail, full) % 8 == 0, "mbarriers are 8-byte aligned");
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
    StatusRef status;
    int M, N, K, cap;
    float threshold;
    int stages;
    int kslice;                          // columns of X per bulk-copied slice
    int kblocks;
    int tiles;
    uint32_t xq_off;                     // byte offset of the quantized X in shared memory
    uint32_t tail_off;
    uint64_t timeout_ns;
};

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8]) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __half22float2(h[e]);
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}

// Byte offset of Xq[m, k0 .. k0+7] (k0 a multiple of 8) in the 128-byte-swizzled K-major
// layout: per 128-column block, 16 rows of 128 bytes in two 8-row atoms of 1024 bytes; the
// 16-byte chunk index within a row is XORed with (row mod 8).
__device__ __forceinline__ uint32_t xq_offset(int m, int k0) {
    const int kb = k0 >> 7, c = k0 & 127;
    return (uint32_t)(kb * (DM * 128) + (m >> 3) * 1024 + (m & 7) * 128 +
                      ((((c >> 4) ^ (m & 7)) << 4) | (c & 15)));
}

__global__ void __launch_bounds__(DTHREADS, 1)
llmint8_decode_kernel(const __grid_constant__ CUtensorMap tmCB, const DArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    DTail *tail = reinterpret_cast<DTail *>(smem + a.tail_off);
    uint8_t *xq = smem + a.xq_off;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int t = threadIdx.x;
    const int S = a.stages;
    const int kpad = a.kblocks * DBK;
    // While the quantization below runs the stage buffers are idle: X is brought there by
    // bulk copies, a column slice of all rows at a time ([row][column] fp16).
    __half *stash = reinterpret_cast<__half *>(smem);
    const int ks = a.kslice;                           // columns per slice (multiple of 128)
    const int nslices = (a.K + ks - 1) / ks;

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
        fence_mbar_init();
        tma_prefetch_desc(&tmCB);
    }
    if (t < DM) tail->rowmax[t] = 0u;
    if (warp == 1) tmem_alloc(smem_addr(&tail->tmem_base), 32);
    // zero the operand (rows >= M and columns >= K must read as 0)
    for (int i = t; i < kpad * DM / 16; i += DTHREADS)
        reinterpret_cast<uint4 *>(xq)[i] = make_uint4(0, 0, 0, 0);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const BoundedWait wait{&tail->abort_flag, a.status, a.timeout_ns};
    uint32_t xphase = 0;
    bool x_ok = true;

    // Copies columns [k0, k0 + width) of every row of X into the stash (one thread issues,
    // everyone waits).  Returns false if the copy did not land in time.
    auto load_slice = [&](int k0, int width) -> bool {
        if (t == 0) {
            const uint32_t bar = smem_addr(&tail->xbar);
            mbar_arrive_expect_tx(bar, (uint32_t)(a.M * width * 2));
            for (int m = 0; m < a.M; ++m)
                bulk_load_1d(smem_addr(stash + m * ks), a.X + (int64_t)m * a.K + k0,
                             (uint32_t)(width * 2), bar);
        }
        int ok = 0;
        if (t == 0) ok = wait(smem_addr(&tail->xbar), xphase) ? 1 : 0;
        xphase ^= 1;
        return __syncthreads_or(ok) != 0;
    };

    // ---------------- phase A: quantize X in this CTA, before the weight stream starts ----
    // (its loads would otherwise queue behind the weight requests of every SM).  Compact,
    // rolled loops: this code runs once per CTA, so its size is paid in instruction fetch.
    for (int sl = 0; sl < nslices && x_ok; ++sl) {
        const int k0 = sl * ks, width = min(ks, a.K - k0), wchunks = width / 8;
        x_ok = load_slice(k0, width);
        if (!x_ok) break;
        // pass 1a: outlier bits of each 8-column chunk (a column is an outlier when any
        // row has |x| >= threshold)
        for (int c = t; c < wchunks; c += DTHREADS) {
            uint32_t fl = 0;
            for (int m = 0; m < a.M; ++m) {
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(stash + m * ks + c * 8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e) fl |= (fabsf(f[e]) >= a.threshold ? 1u : 0u) << e;
            }
            tail->flags[k0 / 8 + c] = (uint8_t)fl;
        }
        __syncthreads();
        // pass 1b: row maxima over the regular columns
        for (int m = 0; m < a.M; ++m) {
            float r = 0.0f;
            for (int c = t; c < wchunks; c += DTHREADS) {
                const uint32_t fl = tail->flags[k0 / 8 + c];
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(stash + m * ks + c * 8), f);
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    if (!((fl >> e) & 1u)) r = fmaxf(r, fabsf(f[e]));
            }
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) r = fmaxf(r, __shfl_xor_sync(0xffffffffu, r, o));
            if (lane == 0) atomicMax(&tail->rowmax[m], __float_as_uint(r));
        }
        fence_proxy_async_smem();   // the next slice's copy overwrites what was just read
        __syncthreads();
    }

    // ascending outlier list (one warp), its count, and the device status of the call
    const int nchunks_all = a.K / 8;
    if (warp == 1) {
        const int per = (nchunks_all + 31) / 32;
        const int c0 = lane * per, c1 = min(nchunks_all, c0 + per);
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
    if (t < DM) {
        const float amax = __uint_as_float(tail->rowmax[t]);
        tail->sca[t] = amax;
        tail->mult[t] = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    }
    __syncthreads();

    // pass 2: int8 rows into the swizzled operand (the last slice is still in the stash)
    for (int sl = nslices - 1; sl >= 0 && x_ok; --sl) {
        const int k0 = sl * ks, width = min(ks, a.K - k0), wchunks = width / 8;
        if (sl != nslices - 1) {
            fence_proxy_async_smem();
            __syncthreads();
            x_ok = load_slice(k0, width);
            if (!x_ok) break;
        }
        for (int i = t; i < a.M * wchunks; i += DTHREADS) {
            const int m = i / wchunks, c = i - m * wchunks;
            const float mul = tail->mult[m];
            if (mul > 0.0f) {
                const uint32_t fl = tail->flags[k0 / 8 + c];
                float f[8];
                unpack8(*reinterpret_cast<const uint4 *>(stash + m * ks + c * 8), f);
                uint32_t lo = 0, hi = 0;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    int q = 0;
                    if (!((fl >> e) & 1u))
                        q = max(-127, min(127, __float2int_rn(__fmul_rn(f[e], mul))));
                    const uint32_t b = (uint32_t)(q & 0xff);
                    if (e < 4) lo |= b << (8 * e);
                    else hi |= b << (8 * (e - 4));
                }
                *reinterpret_cast<uint2 *>(xq + xq_offset(m, k0 + c * 8)) = make_uint2(lo, hi);
            }
        }
    }
    {
        // X at the outlier columns, [j][m]
        const int n_out = tail->n_out;
        for (int i = t; i < n_out * DM; i += DTHREADS) {
            const int j = i / DM, m = i % DM;
            tail->xo[i] = m < a.M ? a.X[(int64_t)m * a.K + tail->idx[j]] : __float2half_rn(0.f);
        }
    }
    // generic-proxy writes (xq) and reads (the stash, about to be overwritten by TMA) must
    // be ordered before the async proxy touches that shared memory
    fence_proxy_async_smem();
    __syncthreads();
    if (!x_ok) {
        // the copy of X timed out (already recorded): nothing valid to compute; let the
        // copy in flight land before the CTA exits
        if (t == 0) drain_wait(smem_addr(&tail->xbar), xphase ^ 1, a.status);
        tc_fence_before();
        __syncthreads();
        if (warp == 1) {
            tc_fence_after();
            tmem_dealloc(tmem, 32);
        }
        return;
    }
    const int n_out = tail->n_out;

    if (warp == 0) {
        // --------------------------------------------------- weight stream (TMA) ----
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, used = 0, last_parity = 0;
            for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
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
    } else if (warp == 1) {
        // ----------------------------------------------------------------- MMA issue ----
        if (lane == 0) {
            const uint32_t idesc = idesc_i8(DBM, DM);
            const uint32_t xq_base = smem_addr(xq);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
                if (!wait(smem_addr(&tail->acc_empty[acc]), acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(acc * DM);
                bool ok = true;
                for (int it = 0; it < a.kblocks; ++it) {
                    const int kb = rotated_kblock(it, tile, a.kblocks);
                    if (!wait(smem_addr(&tail->full[stage]), phase)) {
                        ok = false;
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
                if (!ok) break;
                tc_commit(smem_addr(&tail->acc_full[acc]));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            tc_commit(smem_addr(&tail->mma_done));
            drain_wait(smem_addr(&tail->mma_done), 0, a.status);
        }
    } else if (warp >= 4) {
        // ------------------------------------------------------------------ epilogue ----
        const int q = warp & 3;
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        const float inv = 1.0f / 16129.0f;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = blockIdx.x; tile < a.tiles; tile += gridDim.x) {
            int ok = 0;
            if (lane == 0) ok = wait(smem_addr(&tail->acc_full[acc]), acc_phase) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            uint32_t d[DM];
            tmem_ld_32x16(tl + (uint32_t)(acc * DM), d);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&tail->acc_empty[acc]));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;

            const int n = tile * DBM + q * 32 + lane;
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
                    const uint4 x0 = xv[0], x1 = xv[1];
                    float f0[8], f1[8];
                    unpack8(x0, f0);
                    unpack8(x1, f1);
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
    static bool attr_set[64] = {false};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int sms;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!attr_set[dev]) {
            err = cudaDeviceGetAttribute(&sms_cache[dev], cudaDevAttrMultiProcessorCount, dev);
            if (err != cudaSuccess) return err;
            err = cudaFuncSetAttribute(llmint8_decode_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_LIMIT);
            if (err != cudaSuccess) return err;
            attr_set[dev] = true;
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
    a.status = d.status;
    a.M = (int)d.M;
    a.N = (int)d.N;
    a.K = (int)d.K;
    a.cap = (int)d.cap;
    a.threshold = d.threshold;
    a.kblocks = (int)ceil_div(d.K, DBK);
    a.tiles = (int)ceil_div(d.N, DBM);
    a.timeout_ns = d.timeout_ns;
    // shared memory: [stages][xq][tail], 1024-byte aligned pieces, plus 1 KB alignment slack
    const uint32_t xq_bytes = (uint32_t)(a.kblocks * DBK * DM);
    const uint32_t tail_bytes = (uint32_t)align_up(sizeof(DTail), 1024);
    const int64_t room = SMEM_LIMIT - 1024 - xq_bytes - tail_bytes;
    const int stages = (int)std::min<int64_t>(DMAX_STAGES, room / DSTAGE);
    if (stages < 2) return cudaErrorInvalidValue;
    a.stages = stages;
    {
        // X is brought into the idle stage buffers a column slice of all rows at a time
        const int64_t per_col = 2 * d.M;
        int64_t ks = (int64_t)stages * DSTAGE / per_col;
        a.kslice = (int)(ks >= d.K ? d.K : ks / 128 * 128);
        if (a.kslice < 128 && a.kslice < d.K) return cudaErrorInvalidValue;
    }
    a.xq_off = (uint32_t)(stages * DSTAGE);
    a.tail_off = a.xq_off + xq_bytes;
    const int smem = (int)(a.tail_off + sizeof(DTail) + 1024);

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
    const int grid = std::min(a.tiles, sms);
    llmint8_decode_kernel<<<grid, DTHREADS, smem, s>>>(tm, a);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace llmint8

// Memory-bound kernels of the LLM.int8() layer on sm_100a:
//   outlier_scan      - per-column "some |x| >= threshold" flags, one bitmap word per 32
//                       columns and per row split, written without atomics;
//   outlier_compact   - OR of the row-split bitmaps, ascending index list, count, status;
//   quantize_rows     - row absmax over the regular columns, absmax quantization to int8
//                       (outlier columns zeroed) and the compact gather of the fp16 outlier
//                       columns Xo; the CTAs past the last row gather the fp16 weights of the
//                       outlier columns, Wo[n, j];
//   quantize_weight   - per-output-channel absmax quantization of W (one-time setup);
//   dequant           - (CB * SCB) / 127 back to fp16.
// Rounding follows the definition exactly: multiplier = fl32(127 / absmax) (IEEE division),
// product rounded once to fp32, then round-half-to-even to an integer.
#include "common.cuh"
#include "kernels.h"

namespace llmint8 {

namespace {

constexpr int kThreads = 256;

// Programmatic dependent launch: every kernel of a layer call is launched so that its CTAs
// may start while the previous kernel in the stream finishes.  Each waits for that kernel
// (and so for everything before it) before it touches global memory, and lets the next one
// launch right away.
__device__ __forceinline__ void pdl_wait_then_release() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void unpack8(const uint4 &v, float (&f)[8]) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float2 t = __half22float2(h[e]);
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}

__device__ __forceinline__ int quant1(float x, float s) {
    int q = __float2int_rn(__fmul_rn(x, s));
    return max(-127, min(127, q));
}

__device__ __forceinline__ uint2 quant8(const float (&f)[8], float s, uint32_t skip_mask) {
    uint32_t lo = 0, hi = 0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        int q = ((skip_mask >> e) & 1u) ? 0 : quant1(f[e], s);
        uint32_t b = (uint32_t)(q & 0xff);
        if (e < 4) lo |= b << (8 * e);
        else hi |= b << (8 * (e - 4));
    }
    return make_uint2(lo, hi);
}

__device__ __forceinline__ float block_max(float v, float *red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[warp] = v;
    __syncthreads();
    if (warp == 0) {
        v = lane < (int)(blockDim.x >> 5) ? red[lane] : 0.0f;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
        if (lane == 0) red[0] = v;
    }
    __syncthreads();
    return red[0];
}

// grid (ceil(K/8/256), splits); thread = 8 consecutive columns, loops over its row split.
// Plain cached loads: X is read again right after by the row quantization, from L2 when it
// fits there.
__global__ void __launch_bounds__(kThreads)
outlier_scan_kernel(const __half *__restrict__ X, int64_t M, int64_t K, float threshold,
                    int64_t rows_per_split, uint32_t *__restrict__ partial, int64_t nwords) {
    pdl_wait_then_release();
    const int64_t chunk = (int64_t)blockIdx.x * kThreads + threadIdx.x;
    const int64_t nchunks = K / 8;
    const int64_t r0 = (int64_t)blockIdx.y * rows_per_split;
    const int64_t r1 = min(M, r0 + rows_per_split);
    uint32_t bits = 0;
    if (chunk < nchunks) {
        const uint4 *p = reinterpret_cast<const uint4 *>(X) + r0 * nchunks + chunk;
        int64_t r = r0;
        // eight rows' loads in flight before any use: the scan is bound by bytes in flight
        for (; r + 8 <= r1; r += 8) {
            uint4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldg(p + u * nchunks);
            p += 8 * nchunks;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                float f[8];
                unpack8(v[u], f);
#pragma unroll
                for (int e = 0; e < 8; ++e) bits |= (fabsf(f[e]) >= threshold ? 1u : 0u) << e;
            }
        }
        for (; r < r1; ++r) {
            float f[8];
            unpack8(__ldg(p), f);
            p += nchunks;
#pragma unroll
            for (int e = 0; e < 8; ++e) bits |= (fabsf(f[e]) >= threshold ? 1u : 0u) << e;
        }
    }
    // four neighbouring threads hold the four bytes of one 32-column word
    uint32_t word = bits << (8 * (threadIdx.x & 3));
    word |= __shfl_xor_sync(0xffffffffu, word, 1);
    word |= __shfl_xor_sync(0xffffffffu, word, 2);
    if ((threadIdx.x & 3) == 0 && chunk < nchunks)
        partial[(int64_t)blockIdx.y * nwords + chunk / 4] = word;
}

// One CTA of 1024 threads: OR over the row splits, popcount, exclusive scan, ascending
// index list.  Also writes the workspace status word (resetting it for this call).  The OR
// over the splits is spread over every thread: thread t takes word t % nwords' share of
// the splits when nwords < 1024, and the shares meet in shared memory.  The "splits" may
// also be caller-supplied bitmaps (one per row block of a token-parallel layer): bits at
// columns >= K are dropped, so no index past the last column comes out.
constexpr int kCompactThreads = 1024;
constexpr int kMaxWordsPerThread = 4;   // nwords <= 4096 (K <= 131072)

__global__ void __launch_bounds__(kCompactThreads)
outlier_compact_kernel(const uint32_t *__restrict__ partial, int splits, int64_t nwords,
                       int64_t K, int32_t *__restrict__ idx, int64_t cap,
                       int32_t *__restrict__ count_out, uint32_t *__restrict__ bitmap_out,
                       StatusRef status) {
    pdl_wait_then_release();
    __shared__ int warp_tot[32];
    __shared__ uint32_t merged[kCompactThreads];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    if (nwords < kCompactThreads) {
        // parts of the split range per word
        const int parts = kCompactThreads / (int)nwords;
        const int wi = tid % (int)nwords, part = tid / (int)nwords;
        uint32_t v = 0;
        if (part < parts) {
            const int s0 = (int)((int64_t)splits * part / parts);
            const int s1 = (int)((int64_t)splits * (part + 1) / parts);
            int sp = s0;
            for (; sp + 4 <= s1; sp += 4) {
                const uint32_t a0 = partial[(int64_t)sp * nwords + wi];
                const uint32_t a1 = partial[(int64_t)(sp + 1) * nwords + wi];
                const uint32_t a2 = partial[(int64_t)(sp + 2) * nwords + wi];
                const uint32_t a3 = partial[(int64_t)(sp + 3) * nwords + wi];
                v |= a0 | a1 | a2 | a3;
            }
            for (; sp < s1; ++sp) v |= partial[(int64_t)sp * nwords + wi];
        }
        merged[tid] = v;
        __syncthreads();
        if (tid < nwords) {
            uint32_t o = 0;
            for (int pp = 0; pp < parts; ++pp) o |= merged[pp * (int)nwords + tid];
            merged[tid] = o;      // only threads < nwords write, after every read above
        }
        __syncthreads();
    }
    const int wpt = (int)ceil_div(nwords, kCompactThreads);
    const int64_t w0 = (int64_t)tid * wpt;
    uint32_t w[kMaxWordsPerThread];
    int cnt = 0;
#pragma unroll
    for (int i = 0; i < kMaxWordsPerThread; ++i) {
        w[i] = 0;
        const int64_t wi = w0 + i;
        if (i < wpt && wi < nwords) {
            uint32_t v = 0;
            if (nwords < kCompactThreads) {
                v = merged[wi];
            } else {
                for (int sp = 0; sp < splits; ++sp) v |= partial[(int64_t)sp * nwords + wi];
            }
            if (wi == nwords - 1 && (K & 31) != 0) v &= (1u << (K & 31)) - 1u;
            w[i] = v;
            bitmap_out[wi] = v;
            cnt += __popc(v);
        }
    }
    // block-wide exclusive scan of cnt
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        int v = warp_tot[lane];
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int t = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += t;
        }
        warp_tot[lane] = x - v;   // exclusive prefix of warp totals
    }
    __syncthreads();
    int pos = warp_tot[warp] + incl - cnt;
#pragma unroll
    for (int i = 0; i < kMaxWordsPerThread; ++i) {
        uint32_t v = w[i];
        while (v) {
            const int b = __ffs(v) - 1;
            v &= v - 1;
            LLMINT8_DCHECK((w0 + i) * 32 + b < K, status);
            if (pos < cap) idx[pos] = (int32_t)((w0 + i) * 32 + b);
            ++pos;
        }
    }
    if (tid == kCompactThreads - 1) {
        *count_out = pos;
        status.set(pos > cap ? LLMINT8_ERR_OUTLIER_CAPACITY : LLMINT8_OK);
    }
}

// Weight rows a gather warp takes when the outlier columns are few (at most 64): the loads of
// all of them are issued before any use, and the gather CTAs past the first eighth have no
// rows and exit at once.  With more columns a warp takes one row, so that there are enough
// warps for the longer chains of loads.
constexpr int kGatherRows = 8;

// The fp16 weights of the outlier columns for weight rows n0 .. n0 + rows - 1 (one warp; lane
// j of a pass takes outlier column j).
__device__ __forceinline__ void gather_w_rows(const int8_t *__restrict__ CB,
                                              const float *__restrict__ SCB,
                                              const __half *__restrict__ W16, int64_t n0,
                                              int rows, int64_t N, int64_t K,
                                              const int32_t *__restrict__ idx, int64_t n_o,
                                              int64_t pitch, __half *__restrict__ Wo, int lane) {
    const int64_t n_o64 = align_up(n_o, 64);
    for (int64_t j = lane; j < n_o64; j += 32) {
        const int64_t col = j < n_o ? idx[j] : 0;
        __half v[kGatherRows];
#pragma unroll
        for (int r = 0; r < kGatherRows; ++r) {
            const int64_t n = n0 + r;
            v[r] = __float2half_rn(0.0f);
            if (r < rows && j < n_o && n < N) {
                if (W16 != nullptr)
                    v[r] = W16[n * K + col];
                else
                    v[r] = __float2half_rn(
                        __fdiv_rn(__fmul_rn((float)CB[n * K + col], SCB[n]), 127.0f));
            }
        }
#pragma unroll
        for (int r = 0; r < kGatherRows; ++r)
            if (r < rows && n0 + r < N) Wo[(n0 + r) * pitch + j] = v[r];
    }
}

struct GatherW {
    const int8_t *CB;
    const float *SCB;
    const __half *W16;
    __half *Wo;          // null: no gather
    int64_t N;
};

// Row quantization.  A CTA takes rows_per_cta rows, tpr = 256 / rows_per_cta threads each
// (tpr a power of two, 32 ... 256, chosen so that a thread holds up to kCache 8-column chunks
// of its row in registers); CTAs past the last row block gather Wo, one warp per weight row.
// In packed fp16: the outlier halves of each chunk are cleared with a mask expanded from the
// bitmap byte, the row absmax is a maximum of |x| pairs (exact), and the codes are
// fl32(x * fl32(127 / absmax)) rounded half to even by adding 1.5 * 2^23 (exact for these
// magnitudes), whose low byte is the int8 code.
constexpr int kCache = 8;

// 0xffff in each half of the four words of a chunk whose outlier bit is set in b
__device__ __forceinline__ void chunk_mask(uint32_t b, uint32_t (&m)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e)
        m[e] = (((b >> (2 * e)) & 1u) ? 0x0000ffffu : 0u) |
               (((b >> (2 * e + 1)) & 1u) ? 0xffff0000u : 0u);
}
__device__ __forceinline__ uint32_t hmax2_u32(uint32_t a, uint32_t b) {
    const __half2 r = __hmax2(*reinterpret_cast<const __half2 *>(&a),
                              *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}
// |x| pairs of a chunk with the outlier halves cleared, folded into the running maximum
__device__ __forceinline__ uint32_t chunk_absmax(const uint4 &v, uint32_t skip, uint32_t acc) {
    uint32_t m[4];
    chunk_mask(skip, m);
    acc = hmax2_u32(acc, v.x & 0x7fff7fffu & ~m[0]);
    acc = hmax2_u32(acc, v.y & 0x7fff7fffu & ~m[1]);
    acc = hmax2_u32(acc, v.z & 0x7fff7fffu & ~m[2]);
    acc = hmax2_u32(acc, v.w & 0x7fff7fffu & ~m[3]);
    return acc;
}
// the eight int8 codes of a chunk (0 at the outlier columns, and everywhere when s == 0)
__device__ __forceinline__ uint2 chunk_codes(const uint4 &v, uint32_t skip, float s) {
    uint32_t m[4];
    chunk_mask(skip, m);
    const uint32_t w[4] = {v.x & ~m[0], v.y & ~m[1], v.z & ~m[2], v.w & ~m[3]};
    uint32_t c[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w[e]));
        c[2 * e] = __float_as_uint(__fadd_rn(__fmul_rn(f.x, s), 12582912.0f));
        c[2 * e + 1] = __float_as_uint(__fadd_rn(__fmul_rn(f.y, s), 12582912.0f));
    }
    return make_uint2(__byte_perm(__byte_perm(c[0], c[1], 0x0040), __byte_perm(c[2], c[3], 0x0040),
                                  0x5410),
                      __byte_perm(__byte_perm(c[4], c[5], 0x0040), __byte_perm(c[6], c[7], 0x0040),
                                  0x5410));
}

__global__ void __launch_bounds__(kThreads, 4)
quantize_rows_kernel(const __half *__restrict__ X, int64_t M, int64_t K,
                     const uint32_t *__restrict__ bitmap, const int32_t *__restrict__ idx,
                     const int32_t *__restrict__ count, int64_t cap, int64_t xo_pitch,
                     int8_t *__restrict__ Xq, float *__restrict__ SCA, __half *__restrict__ Xo,
                     int tpr_log2, int64_t row_ctas, const GatherW gw) {
    pdl_wait_then_release();
    __shared__ uint32_t red[kThreads / 32];
    if ((int64_t)blockIdx.x >= row_ctas) {
        const int64_t n_o = min((int64_t)*count, cap);
        const int rows = n_o <= 64 ? kGatherRows : 1;
        const int64_t n0 =
            (((int64_t)blockIdx.x - row_ctas) * (kThreads / 32) + (threadIdx.x >> 5)) * rows;
        if (n0 < gw.N)
            gather_w_rows(gw.CB, gw.SCB, gw.W16, n0, rows, gw.N, K, idx, n_o, xo_pitch, gw.Wo,
                          threadIdx.x & 31);
        return;
    }
    const int tpr = 1 << tpr_log2;
    const int t = threadIdx.x & (tpr - 1);
    const int64_t row = (int64_t)blockIdx.x * (kThreads >> tpr_log2) + (threadIdx.x >> tpr_log2);
    const bool live = row < M;
    const int64_t nchunks = K / 8;
    const uint4 *xr = reinterpret_cast<const uint4 *>(X + (live ? row : 0) * K);
    uint4 cache[kCache];
    uint32_t skipc[kCache / 4] = {};         // the chunks' outlier bytes, four to a word
#pragma unroll
    for (int i = 0; i < kCache; ++i) {       // issue every load before using any
        const int64_t c = t + (int64_t)i * tpr;
        const bool in = live && c < nchunks;
        cache[i] = in ? xr[c] : make_uint4(0, 0, 0, 0);
        if (in) skipc[i / 4] |= ((bitmap[c >> 2] >> ((c & 3) * 8)) & 0xffu) << (8 * (i % 4));
    }
    uint32_t am = 0u;                        // |x| maxima, fp16 pairs
#pragma unroll
    for (int i = 0; i < kCache; ++i)
        am = chunk_absmax(cache[i], (skipc[i / 4] >> (8 * (i % 4))) & 0xffu, am);
    for (int64_t c = t + (int64_t)kCache * tpr; live && c < nchunks; c += tpr)
        am = chunk_absmax(xr[c], (bitmap[c >> 2] >> ((c & 3) * 8)) & 0xffu, am);
    // the row's maximum: over the warp, then over the row's warps
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) am = hmax2_u32(am, __shfl_xor_sync(0xffffffffu, am, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = am;
    __syncthreads();
    const int wpr = tpr >> 5;                // warps per row
    const int w0 = (threadIdx.x >> 5) & ~(wpr - 1);
    for (int w = 0; w < wpr; ++w) am = hmax2_u32(am, red[w0 + w]);
    const __half2 h = *reinterpret_cast<const __half2 *>(&am);
    const float amax = fmaxf(__low2float(h), __high2float(h));
    if (!live) return;
    if (t == 0) SCA[row] = amax;
    const float s = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    uint2 *qr = reinterpret_cast<uint2 *>(Xq + row * K);
#pragma unroll
    for (int i = 0; i < kCache; ++i) {
        const int64_t c = t + (int64_t)i * tpr;
        if (c < nchunks) qr[c] = chunk_codes(cache[i], (skipc[i / 4] >> (8 * (i % 4))) & 0xffu, s);
    }
    for (int64_t c = t + (int64_t)kCache * tpr; c < nchunks; c += tpr)
        qr[c] = chunk_codes(xr[c], (bitmap[c >> 2] >> ((c & 3) * 8)) & 0xffu, s);
    if (Xo != nullptr) {
        const int64_t n_o = min((int64_t)*count, cap);
        const int64_t n_o64 = align_up(n_o, 64);
        const __half *x = X + row * K;
        for (int64_t j = t; j < n_o64; j += tpr)
            Xo[row * xo_pitch + j] = j < n_o ? x[idx[j]] : __float2half_rn(0.0f);
    }
}

// One CTA per output channel n.
__global__ void __launch_bounds__(kThreads)
quantize_weight_kernel(const __half *__restrict__ W, int64_t K, int8_t *__restrict__ CB,
                       float *__restrict__ SCB) {
    __shared__ float red[32];
    const int64_t n = blockIdx.x;
    const int64_t nchunks = K / 8;
    const uint4 *wr = reinterpret_cast<const uint4 *>(W + n * K);
    uint4 cache[kCache];
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < kCache; ++i) {       // issue every load before using any
        const int64_t c = threadIdx.x + (int64_t)i * kThreads;
        cache[i] = c < nchunks ? wr[c] : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < kCache; ++i) {
        const int64_t c = threadIdx.x + (int64_t)i * kThreads;
        if (c < nchunks) {
            float f[8];
            unpack8(cache[i], f);
#pragma unroll
            for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
        }
    }
    for (int64_t c = threadIdx.x + (int64_t)kCache * kThreads; c < nchunks; c += kThreads) {
        float f[8];
        unpack8(wr[c], f);
#pragma unroll
        for (int e = 0; e < 8; ++e) amax = fmaxf(amax, fabsf(f[e]));
    }
    amax = block_max(amax, red);
    if (threadIdx.x == 0) SCB[n] = amax;
    const float s = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    const uint32_t skip = amax > 0.0f ? 0u : 0xffu;
    uint2 *qr = reinterpret_cast<uint2 *>(CB + n * K);
#pragma unroll
    for (int i = 0; i < kCache; ++i) {
        const int64_t c = threadIdx.x + (int64_t)i * kThreads;
        if (c < nchunks) {
            float f[8];
            unpack8(cache[i], f);
            qr[c] = quant8(f, s, skip);
        }
    }
    for (int64_t c = threadIdx.x + (int64_t)kCache * kThreads; c < nchunks; c += kThreads) {
        float f[8];
        unpack8(wr[c], f);
        qr[c] = quant8(f, s, skip);
    }
}

// Grid-stride over 8-element chunks.
__global__ void __launch_bounds__(kThreads)
dequant_kernel(const int8_t *__restrict__ CB, const float *__restrict__ SCB, int64_t N, int64_t K,
               __half *__restrict__ W_out) {
    const int64_t per_row = K / 8;
    const int64_t total = N * per_row;
    for (int64_t c = (int64_t)blockIdx.x * kThreads + threadIdx.x; c < total;
         c += (int64_t)gridDim.x * kThreads) {
        const int64_t n = c / per_row;
        const float scb = SCB[n];
        const uint2 q = reinterpret_cast<const uint2 *>(CB)[c];
        __align__(16) __half out[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const uint32_t word = e < 4 ? q.x : q.y;
            const int v = (int)(int8_t)((word >> (8 * (e & 3))) & 0xffu);
            out[e] = __float2half_rn(__fdiv_rn(__fmul_rn((float)v, scb), 127.0f));
        }
        reinterpret_cast<uint4 *>(W_out)[c] = *reinterpret_cast<const uint4 *>(out);
    }
}

}  // namespace

// ------------------------------------------------------------------ launchers ----------

ScanPlan scan_plan(int64_t M, int64_t K) {
    ScanPlan p;
    p.col_blocks = ceil_div(K / 8, kThreads);
    const int64_t target_ctas = 296;   // two waves' worth of CTAs on a 148-SM part
    int64_t splits = std::max<int64_t>(1, target_ctas / p.col_blocks);
    splits = std::min<int64_t>(splits, M);
    p.rows_per_split = ceil_div(M, splits);
    p.splits = ceil_div(M, p.rows_per_split);
    p.nwords = ceil_div(K, 32);
    return p;
}

namespace {

// Launch with the programmatic-stream-serialization attribute (see pdl_wait_then_release).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t s,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace

cudaError_t launch_outlier_detect(const __half *X, int64_t M, int64_t K, float threshold,
                                  const ScanPlan &plan, uint32_t *partial, uint32_t *bitmap,
                                  int32_t *idx, int64_t cap, int32_t *count, StatusRef status,
                                  cudaStream_t s) {
    dim3 grid((unsigned)plan.col_blocks, (unsigned)plan.splits);
    cudaError_t e = launch_pdl(outlier_scan_kernel, grid, dim3(kThreads), s, X, M, K, threshold,
                               plan.rows_per_split, partial, plan.nwords);
    note_launches(1);
    if (e != cudaSuccess) return e;
    e = launch_pdl(outlier_compact_kernel, dim3(1), dim3(kCompactThreads), s,
                   (const uint32_t *)partial, (int)plan.splits, plan.nwords, K, idx, cap, count,
                   bitmap, status);
    note_launches(1);
    return e;
}

cudaError_t launch_outlier_merge(const uint32_t *bitmaps, int64_t n_bitmaps, int64_t K,
                                 uint32_t *bitmap, int32_t *idx, int64_t cap, int32_t *count,
                                 StatusRef status, cudaStream_t s) {
    const cudaError_t e = launch_pdl(outlier_compact_kernel, dim3(1), dim3(kCompactThreads), s,
                                     bitmaps, (int)n_bitmaps, ceil_div(K, 32), K, idx, cap,
                                     count, bitmap, status);
    note_launches(1);
    return e;
}

cudaError_t launch_quantize_rows(const __half *X, int64_t M, int64_t K, const uint32_t *bitmap,
                                 const int32_t *idx, const int32_t *count, int64_t cap,
                                 int64_t xo_pitch, int8_t *Xq, float *SCA, __half *Xo,
                                 const int8_t *CB, const float *SCB, const __half *W16, int64_t N,
                                 __half *Wo, cudaStream_t s) {
    GatherW gw;
    gw.CB = CB;
    gw.SCB = SCB;
    gw.W16 = W16;
    gw.Wo = Wo;
    gw.N = Wo != nullptr ? N : 0;
    // one weight row per warp, or kGatherRows when the outlier count cannot pass 64 (the
    // kernel takes kGatherRows whenever the count it reads is at most 64)
    const int64_t rows_per_warp = cap <= 64 ? kGatherRows : 1;
    const int64_t gather_ctas = ceil_div(gw.N, (int64_t)(kThreads / 32) * rows_per_warp);
    // threads per row: enough for kCache chunks each, 32 ... 256
    int tpr_log2 = 5;
    while (tpr_log2 < 8 && ((int64_t)kCache << tpr_log2) < K / 8) ++tpr_log2;
    const int64_t row_ctas = ceil_div(M, kThreads >> tpr_log2);
    const cudaError_t e = launch_pdl(quantize_rows_kernel,
                                     dim3((unsigned)(row_ctas + gather_ctas)), dim3(kThreads), s,
                                     X, M, K, bitmap, idx, count, cap, xo_pitch, Xq, SCA, Xo,
                                     tpr_log2, row_ctas, gw);
    note_launches(1);
    return e;
}

cudaError_t launch_quantize_weight(const __half *W, int64_t N, int64_t K, int8_t *CB, float *SCB,
                                   cudaStream_t s) {
    quantize_weight_kernel<<<(unsigned)N, kThreads, 0, s>>>(W, K, CB, SCB);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_dequant(const int8_t *CB, const float *SCB, int64_t N, int64_t K,
                           __half *W_out, cudaStream_t s) {
    const int64_t total = N * (K / 8);
    const unsigned blocks = (unsigned)std::min<int64_t>(ceil_div(total, kThreads), 148 * 16);
    dequant_kernel<<<blocks, kThreads, 0, s>>>(CB, SCB, N, K, W_out);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace llmint8

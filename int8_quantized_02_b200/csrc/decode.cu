// Decode path of the LLM.int8() layer (few activation rows, M <= 16).
//
// At decode sizes the layer is bound by streaming the int8 weight CB from HBM once; the rest
// must hide under that stream.  One kernel per call, one CTA per SM:
//
//   CTAs 0 .. nq-1, the quantizers (nq <= 8): each waits for the previous grid on the stream
//       (X may be its output) and owns a slice of k-blocks.  It copies its columns of X to
//       shared memory, finds their outlier bits (|x| >= threshold in any row) and, per row, the
//       maximum of |x| over its regular columns, and publishes those maxima and its outlier
//       count as call-tagged words.  Reading every quantizer's words gives it the row scales of
//       the whole layer and its place in the ascending outlier list; it writes the int8 codes
//       of its slice as a block of the operand image (K-major, 128-byte swizzle, the layout of
//       the MMA's B operand in shared memory), stores it to the workspace with one bulk copy,
//       lists its outlier columns and releases done[q] with the call number.
//   CTAs nq.., the streamers, each own bands of Rt consecutive weight rows (output channels);
//       Rt = ceil(N / streamers) rounded up to 8 rows (at most 128), so the bands spread evenly
//       over every SM and no streamer waits on another:
//     warp 0      TMA producer: 2-k-block stages of the band through a shared-memory ring, at
//                 most two on their way while X is quantized (a short queue keeps the
//                 quantizers' latency-bound chain fast) and up to four once the MMAs run;
//     warp 2      once every done[q] holds the call number, copies the image blocks into
//                 shared memory with bulk copies (once when they all fit, else through a ring);
//     warps 1, 3  one thread each issues tcgen05.mma kind::i8 with the weight rows as the
//                 128-row operand and an image block as the 16-column operand, D[n, m] = sum_k
//                 CB[n, k] Xq[m, k], into its own int32 TMEM accumulator (alternate stages);
//     warps 4..7  epilogue: while the weights stream, each thread (one output channel n) forms
//                 the fp16 outlier part sum_{j in O} X[m, O_j] * W_o[n, O_j] + bias_n and its
//                 scale; after the last MMA: y = D * SCA_m * SCB_n / 127^2 + that part, and
//                 with a next threshold the outlier bitmap of Y for the next layer.
// Loops are rolled (little code to fetch while the weight stream keeps the memory system
// busy), and K is bound by the quantizers' slices, not by shared memory.  Same method and
// rounding as the GEMM path (LLM.int8() summary, sections الابتكار الثاني and الصورة الكاملة;
// blog sections MatMul 内部 and 用法).  Every wait is bounded.
#include <cudaTypedefs.h>

#include <cstddef>
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace llmint8 {

namespace {

constexpr int DM = kDecodeMaxM;         // activation rows held (MMA N)
constexpr int DMMA_M = 128;             // MMA rows; rows of the MMA past the band are discarded
constexpr int DBK = 128;                // bytes of K per k-block
constexpr int DTHREADS = 256;
constexpr int DWARPS = DTHREADS / 32;
constexpr int DKS = 2;                  // k-blocks per weight stage (one wait, one commit)
constexpr int DMAX_STAGES = 32;
constexpr int DIMG_MAX = 32;            // operand-image stages at most ...
constexpr int DIMG_BYTES = 65536;       // ... and the shared memory they take at most
// k-blocks per quantizer CTA (aim).  Each quantizer phase is bound by latency, not by its
// slice's size, so fewer quantizers mean fewer partials to exchange and more streamers: at
// K = 4096, 4 quantizers (8 k-blocks each) beat 2, 3, 5 and 8 at every batch size measured.
constexpr int QKB = 8;
// Weight stages a streamer keeps on their way: a short queue keeps the quantizers' latency-bound
// chain fast (1 stage starves the stream, 3 or 5 slow the chain; 2 measured best).
constexpr int DINFLIGHT = 2;
constexpr int SMEM_LIMIT = 232448;      // 227 KB opt-in per CTA
// Two MMA issuers per CTA (warps 1 and 3): issuer i takes the weight stages j with
// j % 2 == i of every tile, into its own int32 accumulator of 16 columns; the epilogue adds the
// two (exact).  Measured on B200: one thread issues a 128 x 16 x 32 MMA about every 60 cycles,
// two threads together one every 40 (the tensor pipe's floor for this shape), and a
// tcgen05.commit costs about 150 cycles; with one issuer the k-loop, not HBM, bounded a call.
// Each issuer issues 8 MMAs per wait and per commit.  Accumulators are double-buffered over
// tiles: column (acc * 2 + issuer) * 16.
constexpr uint32_t DTMEM_COLS = 64;

__device__ __forceinline__ void unpack8(const uint4 &v, float *f) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&v);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const float2 t = __half22float2(h[e]);
        f[2 * e] = t.x;
        f[2 * e + 1] = t.y;
    }
}

// Byte offset of Xq[m, c0 ..] (c0 a multiple of 8, < 128) in one k-block of the
// 128-byte-swizzled K-major image: `rows` (16, or 8 when M <= 8) rows of 128 bytes in 8-row
// atoms of 1024 bytes; the 16-byte chunk index within a row is XORed with (row mod 8).  With
// 8 rows the MMA's second 8-row group is one shared all-zero atom after the image ring (see
// image_desc), which halves the ring's shared memory.
__device__ __forceinline__ uint32_t xq_offset(int m, int c0) {
    return (uint32_t)((m >> 3) * 1024 + (m & 7) * 128 + ((((c0 >> 4) ^ (m & 7)) << 4) | (c0 & 15)));
}

__host__ __device__ constexpr int image_rows(int M) { return M <= 8 ? 8 : kDecodeMaxM; }

// Descriptor of an image block at `saddr` (+ k offset) for the 16-column MMA operand: the two
// 8-row groups are `sbo` bytes apart (1024 in a 16-row block; for an 8-row block the distance
// to the zero atom, so that rows 8..15 read as zeros).
__device__ __forceinline__ uint64_t image_desc(uint32_t saddr, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);      // start address / 16
    d |= (uint64_t)1u << 16;                      // leading byte offset (unused, 16 B)
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;  // stride byte offset between 8-row groups
    d |= (uint64_t)1u << 46;                      // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                      // swizzle: 128 B
    return d;
}

// int8 code of x with multiplier s: round_half_even(fl32(x * s)) as the low byte of a float.
// fl32(y + 1.5 * 2^23) for |y| < 2^22 is 1.5 * 2^23 + (y rounded to an integer, ties to
// even), whose low significand bits are that integer in two's complement.  |y| <= 127 here
// (|x| <= absmax of its row and s = fl32(127 / absmax)), so no clamp is ever active.
__device__ __forceinline__ uint32_t code_byte(float x, float s) {
    return __float_as_uint(__fadd_rn(__fmul_rn(x, s), 12582912.0f)) & 0xffu;
}

// Eight codes packed little-endian; a set bit in `skip` gives 0.
__device__ __forceinline__ uint2 quant8(const float *f, float s, uint32_t skip) {
    uint32_t b[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) b[e] = code_byte(((skip >> e) & 1u) ? 0.0f : f[e], s);
    const uint32_t lo = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040),
                                    0x5410);
    const uint32_t hi = __byte_perm(__byte_perm(b[4], b[5], 0x0040), __byte_perm(b[6], b[7], 0x0040),
                                    0x5410);
    return make_uint2(lo, hi);
}

// L2 eviction policy of the weight stream: it is read once per call (evict first).
__device__ __forceinline__ uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_2d_policy(uint32_t dst, const CUtensorMap *tm, int x, int y,
                                                   uint32_t bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar), "l"(pol)
        : "memory");
}

// Shared memory of the quantizer CTA.
constexpr int QMAX_CHUNKS = 256;         // 8-column chunks of a slice (16 k-blocks)
constexpr int QWORDS = kDecodeMaxQuantizers * (DM + 1);
constexpr int QPOLL = (QWORDS + 31) / 32;  // words a polling lane loads per round
struct QShared {
    uint64_t xbar;                       // the slice of X has landed (bulk copies)
    float sca[DM];                       // row absmax over all regular columns
    float mult[DM];                      // fl32(127 / absmax), 0 for an all-zero row
    int wsum[DWARPS];                    // per-warp outlier counts (list scan)
    int ok;                              // every quantizer's partials arrived in time
    int before, total;                   // outliers of the slices before this one; in all
    uint32_t fl[QMAX_CHUNKS];            // outlier bits of each 8-column chunk of the slice
    unsigned long long xp[QWORDS];       // every quantizer's published partials
};
// A quantizer's shared memory: QShared, then its M x w slice of X (fp16, row stride w), then
// the int8 image of its k-blocks.
constexpr int QX_OFF = 4096;
static_assert(sizeof(QShared) <= QX_OFF, "quantizer tables fit before the staged X");

// Shared memory tail of a streamer CTA.
struct DTail {
    uint64_t full[DMAX_STAGES];
    uint64_t empty[DMAX_STAGES];
    uint64_t ifull[DIMG_MAX];            // an image stage has landed
    uint64_t iempty[DIMG_MAX];           // ... and been consumed by the MMAs
    uint64_t acc_full[2];                // both issuers (one when a tile has one stage) are done
    uint64_t acc_empty[2];
    uint64_t mma_done[2];
    uint64_t tbar;                       // the quantizer's table is published (one poller)
    uint32_t tmem_base;
    int abort_flag;
    int streaming;                       // the MMAs run: the producer may keep more in flight
    int32_t idx[kDecodeMaxOutliers];     // outlier columns, ascending (epilogue copy)
};
static_assert(offsetof(DTail, acc_full) % 8 == 0, "mbarriers are 8-byte aligned");

struct DArgs {
    const __half *X;
    const int8_t *CB;
    const float *SCB;
    const __half *W16;
    const __half *bias;
    __half *Y;
    int32_t *C_debug;
    __half *Wo;                          // [N, wo_pitch] or null
    int64_t wo_pitch;
    const uint32_t *bitmaps;             // [n_bitmaps][ceil(K/32)] given outlier set, or null
    int n_bitmaps;
    uint32_t *ybits;                     // [ceil(N/32)] outlier bitmap of Y for the next
                                         // layer, or null
    float ytf;                           // its threshold on the fp32 value
    int ybits_all;                       // threshold <= 0: every column
    int ncols32;                         // 32 * ceil(N / 32): the columns the bitmap covers
    int32_t *count;
    DecodeTable *table;                  // workspace: what the quantizer publishes
    uint8_t *image;                      // workspace: the int8 operand image, block by block
    StatusRef status;
    unsigned long long epoch;
    int M, N, K, cap;
    float threshold;
    uint32_t thr2;                       // the threshold rounded up to fp16, in both halves:
                                         // for an fp16 x, |x| >= threshold iff |x| >= that
    int rows;                            // image rows: 16, or 8 when M <= 8
    int Rt;                              // weight rows per tile (band)
    int tiles, kblocks, stages;
    int inflight;                        // weight stages on their way at most
    int nq, bpq;                         // quantizer CTAs, k-blocks per quantizer
    int nst;                             // weight stages per tile: ceil(kblocks / DKS)
    int nistage;                         // operand-image stages (DKS blocks each) of a streamer
    int resident;                        // the image stages hold every k-block: filled once
    uint32_t tail_off, xo_off, ring_off; // byte offsets in shared memory (image ring at 0)
    uint64_t timeout_ns;
};

// ------------------------------------------------------------------ the quantizers ----------
// Quantizer q (CTA q < nq) owns the k-blocks [q * bpq, (q + 1) * bpq), a slice of w columns.
// It copies its slice of X to shared memory (one bulk copy per row) and finds there the outlier
// bits of every 8-column chunk (an OR over the rows of |x| >= threshold, packed fp16 compares,
// exact) and, per row, the maximum of |x| over the slice's regular columns.  It publishes those
// maxima and its outlier count as call-tagged words, reads every quantizer's, and so knows the
// row scales of the whole layer and where its outlier columns go in the ascending list.  Then
// it writes the int8 codes of its slice into a shared-memory image, k-block by k-block in the
// layout the streamers copy into their own shared memory, stores the image to the workspace
// with one bulk copy, lists its outlier columns, and releases done[q].
__device__ __forceinline__ void bulk_store_1d(void *dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(src), "r"(bytes)
                 : "memory");
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_store_wait() {
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void release_word(unsigned long long *w, unsigned long long v) {
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(w), "l"(v) : "memory");
}
__device__ __forceinline__ void relaxed_store(unsigned long long *w, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(w), "l"(v) : "memory");
}
__device__ __forceinline__ unsigned long long relaxed_load(const unsigned long long *w) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(w) : "memory");
    return v;
}
// Bounded, backed-off poll by one thread until each of the n <= kDecodeMaxQuantizers words
// holds v.  Each round loads the words together (relaxed); the fence after the round that
// finds them all makes this thread acquire what their writers released.  False, with the
// timeout recorded, when they do not all arrive in time or the CTA is winding down.
__device__ bool poll_all(const unsigned long long *w, int n, unsigned long long v,
                         StatusRef status, uint64_t timeout_ns, volatile int *abort_flag) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        bool ok = true;
#pragma unroll
        for (int j = 0; j < kDecodeMaxQuantizers; ++j)
            if (j < n) ok = (relaxed_load(w + j) == v) && ok;
        if (ok) {
            asm volatile("fence.acq_rel.gpu;" ::: "memory");
            return true;
        }
        __nanosleep(32);
        if ((it & 15u) == 15u) {
            if (*abort_flag) return false;
            if (global_timer_ns() - t0 > timeout_ns) {
                *abort_flag = 1;
                status.timed_out();
                return false;
            }
        }
    }
}

// Stage j of a tile covers k-blocks DKS * sj ..., sj = j rotated by this offset, so that the
// CTAs streaming at the same moment read different column ranges of the 2^n-strided rows.
__device__ __forceinline__ int stage_rot(int tile, int nst) {
    return (int)(((unsigned)tile * 7u) % (unsigned)nst);
}

// 0xffff in each half of the four words of a chunk whose outlier bit is set in b
__device__ __forceinline__ void expand_bits(uint32_t b, uint32_t (&col)[4]) {
#pragma unroll
    for (int e = 0; e < 4; ++e)
        col[e] = (((b >> (2 * e)) & 1u) ? 0x0000ffffu : 0u) |
                 (((b >> (2 * e + 1)) & 1u) ? 0xffff0000u : 0u);
}

__device__ void quantize_x(const DArgs &a, uint8_t *smem) {
    QShared *q = reinterpret_cast<QShared *>(smem);
    const int qi = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kb0 = qi * a.bpq, kb1 = min(a.kblocks, kb0 + a.bpq);
    const int c0 = kb0 * DBK;
    const int w = min(a.K, kb1 * DBK) - c0;               // columns of the slice (16 | w)
    const int nch = w / 8;
    uint8_t *xs = smem + QX_OFF;                          // [M][w] fp16
    uint8_t *is = xs + (size_t)a.M * a.bpq * DBK * 2;     // image of the slice's k-blocks
    const unsigned long long tag = (unsigned long long)(uint32_t)a.epoch << 32;
    const int nwords = (a.K + 31) / 32;

    if (threadIdx.x == 0) {
        const uint32_t xbar = smem_addr(&q->xbar);
        mbar_arrive_expect_tx(xbar, (uint32_t)(a.M * w * 2));
        for (int m = 0; m < a.M; ++m)
            bulk_load_1d(smem_addr(xs + (size_t)m * w * 2), a.X + (int64_t)m * a.K + c0,
                         (uint32_t)(w * 2), xbar);
    }
    for (int c = threadIdx.x; c < nch; c += DTHREADS) q->fl[c] = 0u;
    __syncthreads();
    if (!drain_wait(smem_addr(&q->xbar), 0, a.status)) return;

    // outlier bits: thread t takes chunk t % nch and the rows congruent to t / nch
    if (a.bitmaps) {
        for (int c = threadIdx.x; c < nch; c += DTHREADS) {
            const int cg = c0 / 8 + c;
            uint32_t wd = 0;
            for (int r = 0; r < a.n_bitmaps; ++r)
                wd |= __ldg(a.bitmaps + (int64_t)r * nwords + (cg >> 2));
            q->fl[c] = (wd >> ((cg & 3) * 8)) & 0xffu;
        }
    } else {
        const int rg = max(1, min(a.M, DTHREADS / nch));  // row groups
        if ((int)threadIdx.x < rg * nch) {
            const int c = threadIdx.x % nch;
            uint32_t col[4] = {0u, 0u, 0u, 0u};
#pragma unroll 4
            for (int m = threadIdx.x / nch; m < a.M; m += rg) {
                const uint4 v = *reinterpret_cast<const uint4 *>(xs + ((size_t)m * w + c * 8) * 2);
                col[0] |= hge2_bits(habs2_bits(v.x), a.thr2);
                col[1] |= hge2_bits(habs2_bits(v.y), a.thr2);
                col[2] |= hge2_bits(habs2_bits(v.z), a.thr2);
                col[3] |= hge2_bits(habs2_bits(v.w), a.thr2);
            }
            uint32_t b = 0;
#pragma unroll
            for (int e = 0; e < 4; ++e)
                b |= ((col[e] & 1u) << (2 * e)) | ((col[e] >> 16 & 1u) << (2 * e + 1));
            if (b) atomicOr(&q->fl[c], b);
        }
    }
    __syncthreads();

    // row maxima over the slice's regular columns (warp w: rows w and w + 8); lane 0 publishes
    // each as a tagged word
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        const int m = warp + 8 * r;
        if (m >= a.M) break;                                  // uniform over the warp
        uint32_t rm = 0u;
#pragma unroll 4
        for (int c = lane; c < nch; c += 32) {
            const uint4 v = *reinterpret_cast<const uint4 *>(xs + ((size_t)m * w + c * 8) * 2);
            uint32_t col[4];
            expand_bits(q->fl[c], col);
            rm = hmax2_bits(rm, habs2_bits(v.x) & ~col[0]);
            rm = hmax2_bits(rm, habs2_bits(v.y) & ~col[1]);
            rm = hmax2_bits(rm, habs2_bits(v.z) & ~col[2]);
            rm = hmax2_bits(rm, habs2_bits(v.w) & ~col[3]);
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) rm = hmax2_bits(rm, __shfl_xor_sync(0xffffffffu, rm, o));
        if (lane == 0) {
            const __half2 h = *reinterpret_cast<const __half2 *>(&rm);
            const float amax = fmaxf(__low2float(h), __high2float(h));
            relaxed_store(&a.table->part[qi][m], tag | __float_as_uint(amax));
        }
    }

    // this slice's outlier count (published too) and each thread's position within the
    // slice's list
    const int cpt = (nch + DTHREADS - 1) / DTHREADS;
    const int l0 = min(nch, (int)threadIdx.x * cpt), l1 = min(nch, l0 + cpt);
    int cnt = 0;
    for (int c = l0; c < l1; ++c) cnt += __popc(q->fl[c]);
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    if (lane == 31) q->wsum[warp] = incl;
    __syncthreads();
    int before = 0, mine = 0;
    for (int wi = 0; wi < DWARPS; ++wi) {
        const int sm = q->wsum[wi];
        before += wi < warp ? sm : 0;
        mine += sm;
    }
    before += incl - cnt;
    if (threadIdx.x == 0) relaxed_store(&a.table->part[qi][DM], tag | (uint32_t)mine);

    // every quantizer's partials: words (j, m < M) and (j, DM).  Warp 0 polls; lane i loads
    // words i, i + 32, ... together each round.
    if (warp == 0) {
        const int per = a.M + 1, n = a.nq * per;
        const unsigned long long *src[QPOLL];
        int dst[QPOLL];
#pragma unroll
        for (int k = 0; k < QPOLL; ++k) {
            const int i = min(lane + 32 * k, n - 1);
            const int j = i / per, mm = i - j * per == a.M ? DM : i - j * per;
            src[k] = &a.table->part[j][mm];
            dst[k] = j * (DM + 1) + mm;
        }
        const uint64_t t0 = global_timer_ns();
        bool ok = false;
        for (uint32_t it = 0;; ++it) {
            unsigned long long v[QPOLL];
#pragma unroll
            for (int k = 0; k < QPOLL; ++k) v[k] = relaxed_load(src[k]);
            bool all = true;
#pragma unroll
            for (int k = 0; k < QPOLL; ++k) all = all && (v[k] & 0xffffffff00000000ull) == tag;
            if (__all_sync(0xffffffffu, all)) {
#pragma unroll
                for (int k = 0; k < QPOLL; ++k) q->xp[dst[k]] = v[k];
                ok = true;
                break;
            }
            __nanosleep(32);
            if ((it & 15u) == 15u &&
                __shfl_sync(0xffffffffu, global_timer_ns() - t0 > a.timeout_ns ? 1 : 0, 0)) {
                break;
            }
        }
        if (!ok && lane == 0) a.status.timed_out();
        if (lane == 0) q->ok = ok ? 1 : 0;
    }
    __syncthreads();
    if (!q->ok) return;                                   // timed out (uniform)
    if (threadIdx.x < DM) {
        float amax = 0.0f;
        if ((int)threadIdx.x < a.M)
            for (int j = 0; j < a.nq; ++j)
                amax = fmaxf(amax, __uint_as_float((uint32_t)q->xp[j * (DM + 1) + threadIdx.x]));
        q->sca[threadIdx.x] = amax;
        q->mult[threadIdx.x] = amax > 0.0f ? __fdiv_rn(127.0f, amax) : 0.0f;
    } else if (threadIdx.x == DM) {
        int bq = 0, tot = 0;
        for (int j = 0; j < a.nq; ++j) {
            const int cj = (int)(uint32_t)q->xp[j * (DM + 1) + DM];
            bq += j < qi ? cj : 0;
            tot += cj;
        }
        q->before = bq;
        q->total = tot;
    }
    __syncthreads();

    // the image of the slice; item (block, 16-column group, row) -> 16 codes, one 16-byte store
    const uint32_t blk_bytes = (uint32_t)a.rows * DBK;
    const int nblk = kb1 - kb0;
#pragma unroll 2
    for (int i = threadIdx.x; i < nblk * 8 * a.rows; i += DTHREADS) {
        const int grp = i & 7, m = (i >> 3) % a.rows, blk = (i >> 3) / a.rows;
        uint4 code = make_uint4(0, 0, 0, 0);
        if (m < a.M) {
            const int cl = blk * 16 + grp * 2;             // chunk within the slice
            const uint32_t b0 = cl * 8 < w ? q->fl[cl] : 0xffu;
            const uint32_t b1 = cl * 8 + 8 < w ? q->fl[cl + 1] : 0xffu;
            const uint4 *src = reinterpret_cast<const uint4 *>(xs + ((size_t)m * w + cl * 8) * 2);
            const uint4 v0 = cl * 8 < w ? src[0] : make_uint4(0, 0, 0, 0);
            const uint4 v1 = cl * 8 + 8 < w ? src[1] : make_uint4(0, 0, 0, 0);
            float f[8];
            unpack8(v0, f);
            const uint2 lo = quant8(f, q->mult[m], b0);
            unpack8(v1, f);
            const uint2 hi = quant8(f, q->mult[m], b1);
            code = make_uint4(lo.x, lo.y, hi.x, hi.y);
        }
        *reinterpret_cast<uint4 *>(is + blk * blk_bytes + xq_offset(m, grp * 16)) = code;
    }
    // the image is read by the bulk store (async proxy)
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0)
        bulk_store_1d(a.image + (size_t)kb0 * blk_bytes, smem_addr(is), (uint32_t)nblk * blk_bytes);

    // this slice's entries of the ascending outlier list; quantizer 0 also the row scales and
    // the counts
    int pos = q->before + before;
    for (int c = l0; c < l1; ++c) {
        uint32_t b = q->fl[c];
        while (b) {
            const int e = __ffs(b) - 1;
            b &= b - 1;
            LLMINT8_DCHECK(c0 + c * 8 + e < a.K, a.status);
            if (pos < a.cap) a.table->idx[pos] = c0 + c * 8 + e;
            ++pos;
        }
    }
    if (qi == 0) {
        if (threadIdx.x < DM) a.table->sca[threadIdx.x] = q->sca[threadIdx.x];
        if (threadIdx.x == DM) {
            const int total = q->total;
            a.table->total = total;
            a.table->n_out = min(total, a.cap);
            *a.count = total;
            a.status.set(total > a.cap ? LLMINT8_ERR_OUTLIER_CAPACITY : LLMINT8_OK);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        bulk_store_wait();
        fence_proxy_async_global();
        release_word(&a.table->done[qi], a.epoch);
    }
}

__global__ void __launch_bounds__(DTHREADS, 1)
llmint8_decode_kernel(const __grid_constant__ CUtensorMap tmCB, const DArgs a) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if ((int)blockIdx.x < a.nq) {
        // the next call's kernel may launch now; this one waits for the previous grid before it
        // reads X or writes the workspace
        asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
        if (threadIdx.x == 0) {
            mbar_init(smem_addr(&reinterpret_cast<QShared *>(smem)->xbar), 1);
            fence_mbar_init();
        }
        asm volatile("griddepcontrol.wait;" ::: "memory");
        quantize_x(a, smem);
        return;
    }

    uint8_t *img = smem;                          // nistage x DKS blocks (+ zero atom)
    DTail *tail = reinterpret_cast<DTail *>(smem + a.tail_off);
    __half *xo = reinterpret_cast<__half *>(smem + a.xo_off);     // [j][m]
    uint8_t *ring = smem + a.ring_off;
    const int S = a.stages;
    const uint32_t stage_bytes = (uint32_t)DKS * a.Rt * DBK;
    const uint32_t img_bytes = (uint32_t)a.rows * DBK;            // one k-block of the image
    const int band0 = blockIdx.x - a.nq, bands = gridDim.x - a.nq;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(smem_addr(&tail->full[s]), 1);
            mbar_init(smem_addr(&tail->empty[s]), 1);
        }
        for (int s = 0; s < a.nistage; ++s) {
            mbar_init(smem_addr(&tail->ifull[s]), 1);
            mbar_init(smem_addr(&tail->iempty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&tail->acc_full[s]), a.nst >= 2 ? 2 : 1);
            mbar_init(smem_addr(&tail->acc_empty[s]), 4);
            mbar_init(smem_addr(&tail->mma_done[s]), 1);
        }
        mbar_init(smem_addr(&tail->tbar), 1);
        tail->abort_flag = 0;
        tail->streaming = 0;
        fence_mbar_init();
        tma_prefetch_desc(&tmCB);
    }
    if (warp == 1) tmem_alloc(smem_addr(&tail->tmem_base), DTMEM_COLS);
    // the next call's kernel may launch now (it waits for this grid before it reads or
    // writes anything); this one waits for the previous grid before it touches memory
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const BoundedWait wait{&tail->abort_flag, a.status, a.timeout_ns};

    // stage j of a tile: k-blocks DKS * sj .. (sj rotated by stage_rot; the last stage may hold
    // a single k-block)
    const uint32_t kbox = (uint32_t)a.Rt * DBK;                  // one k-block of the band
    auto rot_of = [&](int tile) { return stage_rot(tile, a.nst); };

    if (warp == 0) {
        // --------------------------------------------------- weight stream (TMA) ----
        if (lane == 0) {
            const uint64_t once = policy_evict_first();
            int stage = 0, issued = 0;
            uint32_t phase = 0, used = 0, last_parity = 0;
            for (int tile = band0; tile < a.tiles; tile += bands) {
                const int rot = rot_of(tile);
                for (int j = 0; j < a.nst; ++j) {
                    int sj = j + rot;
                    if (sj >= a.nst) sj -= a.nst;
                    const int kb0 = sj * DKS, nkb = min(DKS, a.kblocks - kb0);
                    // at most `inflight` stages on their way while X is quantized: a short
                    // memory queue keeps the latency of everything else on the GPU (X, the
                    // tables, the image) low; once the MMAs run, up to four (fewer than the
                    // ring's stages, so the stage waited on is still that use's)
                    const int depth = *reinterpret_cast<volatile int *>(&tail->streaming)
                                          ? min(4, S - 1) : a.inflight;
                    if (issued >= depth) {
                        const int prev = issued - depth;
                        if (!wait(smem_addr(&tail->full[prev % S]), (uint32_t)(prev / S) & 1u))
                            goto drain;
                    }
                    ++issued;
                    if (!wait(smem_addr(&tail->empty[stage]), phase ^ 1)) goto drain;
                    const uint32_t full = smem_addr(&tail->full[stage]);
                    mbar_arrive_expect_tx(full, (uint32_t)nkb * kbox);
                    for (int h = 0; h < nkb; ++h)
                        tma_load_2d_policy(smem_addr(ring + stage * stage_bytes + h * kbox), &tmCB,
                                           (kb0 + h) * DBK, tile * a.Rt, full, once);
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
    } else if (warp == 1 || warp == 3) {
        // ------------------------------------------------------------- MMA issue ----
        const int issuer = warp == 1 ? 0 : 1;
        if (lane == 0 && (issuer == 0 || a.nst >= 2)) {
            const uint32_t idesc = idesc_i8(DMMA_M, DM);
            const uint32_t img_base = smem_addr(img);
            const uint32_t ring_base = smem_addr(ring);
            const uint32_t zero_atom = img_base + (uint32_t)a.nistage * DKS * img_bytes;
            int acc = 0, tl_ = 0;                          // tl_: this CTA's tile count so far
            uint32_t acc_phase = 0;
            bool good = true;
            for (int tile = band0; good && tile < a.tiles; tile += bands, ++tl_) {
                if (!wait(smem_addr(&tail->acc_empty[acc]), acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)((acc * 2 + issuer) * DM);
                const int rot = rot_of(tile);
                bool first = true;
                for (int j = issuer; j < a.nst; j += 2) {
                    const int g = tl_ * a.nst + j;               // stage in the producer's order
                    const int stage = g % S;
                    const uint32_t phase = (uint32_t)(g / S) & 1u;
                    int sj = j + rot;
                    if (sj >= a.nst) sj -= a.nst;
                    const int nkb = min(DKS, a.kblocks - sj * DKS);
                    // the image stage of these k-blocks: fixed when resident, else a ring
                    const int ist = a.resident ? sj : g % a.nistage;
                    const uint32_t ipar = a.resident ? 0u : (uint32_t)(g / a.nistage) & 1u;
                    if (!wait(smem_addr(&tail->ifull[ist]), ipar) ||
                        !wait(smem_addr(&tail->full[stage]), phase)) {
                        good = false;
                        break;
                    }
                    if (issuer == 0) *reinterpret_cast<volatile int *>(&tail->streaming) = 1;
                    tc_fence_after();
                    for (int h = 0; h < nkb; ++h) {
                        const uint32_t sa = ring_base + (uint32_t)stage * stage_bytes + h * kbox;
                        const uint32_t sb = img_base + (uint32_t)(ist * DKS + h) * img_bytes;
                        const uint64_t adesc = sw128_desc(sa);
                        const uint64_t bdesc = image_desc(sb, a.rows == 8 ? zero_atom - sb : 1024u);
#pragma unroll
                        for (int k = 0; k < DBK / 32; ++k) {
                            mma_i8(d, adesc + (uint64_t)(2 * k), bdesc + (uint64_t)(2 * k), idesc,
                                   first ? 0u : 1u);
                            first = false;
                        }
                    }
                    tc_commit(smem_addr(&tail->empty[stage]));
                    if (!a.resident) tc_commit(smem_addr(&tail->iempty[ist]));
                }
                if (!good) break;
                tc_commit(smem_addr(&tail->acc_full[acc]));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1;
            }
            tc_commit(smem_addr(&tail->mma_done[issuer]));
            drain_wait(smem_addr(&tail->mma_done[issuer]), 0, a.status);
        }
    } else if (warp == 2) {
        // ------------------------------------------------- operand image of X, by k-block ----
        // Once the quantizer has published, one thread copies the image blocks (rows x 128
        // bytes each) from the workspace: when every k-block fits (resident), each once, into
        // the image stage of its weight stage; otherwise through a ring of image stages, in
        // the order the MMAs consume them.
        if (a.rows == 8) {
            // the zero atom read as rows 8..15 of an 8-row image block
            for (int i = lane; i < 64; i += 32)
                reinterpret_cast<uint4 *>(img + a.nistage * DKS * img_bytes)[i] =
                    make_uint4(0, 0, 0, 0);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
        if (lane == 0 &&
            poll_all(a.table->done, a.nq, a.epoch, a.status, a.timeout_ns, &tail->abort_flag)) {
            fence_proxy_async_global();           // the image is read by the async proxy
            const int ntiles = (a.tiles - band0 + bands - 1) / bands;   // tiles of this CTA
            const int nstg = a.resident ? a.nst : ntiles * a.nst;
            uint32_t used = 0, last_parity = 0;
            for (int g = 0; g < nstg; ++g) {
                const int tile = band0 + (g / a.nst) * bands;
                int sj = g % a.nst + rot_of(tile);
                if (sj >= a.nst) sj -= a.nst;
                const int kb0 = sj * DKS, nkb = min(DKS, a.kblocks - kb0);
                const int ist = a.resident ? sj : g % a.nistage;
                const uint32_t ipar = a.resident ? 0u : (uint32_t)(g / a.nistage) & 1u;
                if (!a.resident && !wait(smem_addr(&tail->iempty[ist]), ipar ^ 1)) break;
                const uint32_t full = smem_addr(&tail->ifull[ist]);
                mbar_arrive_expect_tx(full, (uint32_t)nkb * img_bytes);
                for (int h = 0; h < nkb; ++h)
                    bulk_load_1d(smem_addr(img + (ist * DKS + h) * img_bytes),
                                 a.image + (size_t)(kb0 + h) * img_bytes, img_bytes, full);
                used |= 1u << ist;
                last_parity = (last_parity & ~(1u << ist)) | (ipar << ist);
            }
            // every copy lands before the CTA may exit
            for (int sl = 0; sl < 32; ++sl)
                if (used & (1u << sl))
                    drain_wait(smem_addr(&tail->ifull[sl]), (last_parity >> sl) & 1u, a.status);
        }
    } else {
        // ------------------------------------------------------------------ epilogue ----
        // Everything of an output channel except the int8 product - its scale, bias and fp16
        // outlier part - is computed while the MMAs still stream the weights; after the last
        // MMA of a tile only the accumulator read, one FMA per value and the stores remain.
        const int qd = warp & 3;
        const int et = threadIdx.x - 128;                 // 0..127 over the epilogue warps
        const uint32_t tl = tmem + ((uint32_t)(qd * 32) << 16);
        const float inv = 1.0f / 16129.0f;
        // one thread polls the quantizers' done words (acquiring what they wrote) and arrives
        // on tbar; lane 0 of each epilogue warp acquires that by its wait on tbar, and the
        // __syncwarp orders it before the reads of its other lanes
        if (et == 0 &&
            poll_all(a.table->done, a.nq, a.epoch, a.status, a.timeout_ns, &tail->abort_flag))
            mbar_arrive(smem_addr(&tail->tbar));
        int ok = 0;
        if (lane == 0) ok = wait(smem_addr(&tail->tbar), 0) ? 1 : 0;
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();
        const int n_out = ok ? a.table->n_out : 0;
        float sca[DM];
#pragma unroll
        for (int mm = 0; mm < DM; ++mm) sca[mm] = ok ? a.table->sca[mm] : 0.0f;
        // the outlier columns and X at them (a 16-row [j][m] table; rows >= M hold 0)
        LLMINT8_DCHECK(n_out >= 0 && n_out <= a.cap, a.status);
        for (int i = et; i < n_out; i += 128) {
            tail->idx[i] = a.table->idx[i];
            LLMINT8_DCHECK(tail->idx[i] >= 0 && tail->idx[i] < a.K, a.status);
        }
        for (int i = et; i < n_out * DM; i += 128) {
            const int j = i / DM, mm = i % DM;
            xo[i] = mm < a.M ? a.X[(int64_t)mm * a.K + a.table->idx[j]] : __float2half_rn(0.0f);
        }
        named_barrier(1, 128);
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int tile = band0; ok && tile < a.tiles; tile += bands) {
            const int r = qd * 32 + lane;                 // TMEM lane = row of the band
            const int n = tile * a.Rt + r;
            const bool live = r < a.Rt && n < a.N;
            float o[DM];
            float scale = 0.0f;
#pragma unroll
            for (int mm = 0; mm < DM; ++mm) o[mm] = 0.0f;
            if (live) {
                const float sb = a.SCB[n];
                const float b = a.bias ? __half2float(a.bias[n]) : 0.0f;
                scale = sb * inv;
                const int8_t *cbrow = a.CB + (int64_t)n * a.K;
                const __half *wrow = a.W16 ? a.W16 + (int64_t)n * a.K : nullptr;
                for (int j0 = 0; j0 < n_out; j0 += 8) {
                    // eight independent loads of the outlier weights before any use
                    int8_t cb8[8];
                    __half w8[8];
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int col = tail->idx[min(j0 + u, n_out - 1)];
                        if (wrow) w8[u] = wrow[col];
                        else cb8[u] = cbrow[col];
                    }
#pragma unroll
                    for (int u = 0; u < 8; ++u) {
                        const int j = j0 + u;
                        if (j >= n_out) break;
                        const __half wh = wrow ? w8[u]
                                               : __float2half_rn(__fdiv_rn(
                                                     __fmul_rn((float)cb8[u], sb), 127.0f));
                        if (a.Wo) a.Wo[(int64_t)n * a.wo_pitch + j] = wh;
                        const float w = __half2float(wh);
                        const uint4 *xv = reinterpret_cast<const uint4 *>(xo + j * DM);
                        float f0[8], f1[8];
                        unpack8(xv[0], f0);
                        unpack8(xv[1], f1);
#pragma unroll
                        for (int mm = 0; mm < 8; ++mm) {
                            o[mm] = fmaf(f0[mm], w, o[mm]);
                            o[mm + 8] = fmaf(f1[mm], w, o[mm + 8]);
                        }
                    }
                }
#pragma unroll
                for (int mm = 0; mm < DM; ++mm) o[mm] += b;
            }
            int okw = 0;
            if (lane == 0) okw = wait(smem_addr(&tail->acc_full[acc]), acc_phase) ? 1 : 0;
            okw = __shfl_sync(0xffffffffu, okw, 0);
            if (!okw) break;
            tc_fence_after();
            uint32_t d[DM];
            tmem_ld_32x16(tl + (uint32_t)(acc * 2 * DM), d);
            if (a.nst >= 2) {
                uint32_t e[DM];
                tmem_ld_32x16(tl + (uint32_t)((acc * 2 + 1) * DM), e);
                tmem_wait_ld();
#pragma unroll
                for (int mm = 0; mm < DM; ++mm) d[mm] += e[mm];
            }
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(smem_addr(&tail->acc_empty[acc]));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1;
            bool yflag = false;   // some |fp16 Y[m, n]| >= the next layer's threshold
            if (live) {
#pragma unroll
                for (int mm = 0; mm < DM; ++mm) {
                    if (mm < a.M) {
                        const float y = fmaf((float)(int32_t)d[mm], sca[mm] * scale, o[mm]);
                        LLMINT8_DCHECK(mm < a.M && n < a.N, a.status);
                        a.Y[(int64_t)mm * a.N + n] = __float2half_rn(y);
                        if (a.C_debug) a.C_debug[(int64_t)mm * a.N + n] = (int32_t)d[mm];
                        // |fp16(y)| >= the next threshold <=> |y| >= ytf
                        yflag = yflag || a.ybits_all || fabsf(y) >= a.ytf;
                    }
                }
            }
            if (a.ybits) {
                // this warp's columns of the band (and any past N, which read as 0) are its own
                // bits of the one or two words they straddle (bands need not start on a
                // multiple of 32): clear those to be 0, then set those to be 1, so the bitmap
                // needs no clearing first and the other bits of a shared word are untouched
                const uint32_t bal = __ballot_sync(0xffffffffu, yflag);
                const uint32_t own =
                    __ballot_sync(0xffffffffu, (live || n >= a.N) && n < a.ncols32);
                const int c0 = tile * a.Rt + qd * 32, sh = c0 & 31;
                if (lane == 0 && own) {
                    uint32_t *w0 = a.ybits + (c0 >> 5);
                    if (own << sh) {
                        atomicAnd(w0, ~((own & ~bal) << sh));
                        if (bal << sh) atomicOr(w0, bal << sh);
                    }
                    if (sh && (own >> (32 - sh))) {
                        atomicAnd(w0 + 1, ~((own & ~bal) >> (32 - sh)));
                        if (bal >> (32 - sh)) atomicOr(w0 + 1, bal >> (32 - sh));
                    }
                }
                // the last word's bits past N, which no band's lanes may reach when the bands
                // are wide: no one sets them, so one AND clears them
                if (tile == a.tiles - 1 && qd == 0 && lane == 0 && (a.N & 31))
                    atomicAnd(a.ybits + (a.N >> 5), (1u << (a.N & 31)) - 1u);
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

DecodePlan decode_plan(int64_t M, int64_t N, int64_t K, int64_t cap, int sms) {
    DecodePlan p;
    const int64_t kblocks = ceil_div(K, DBK);
    p.nq = (int)std::min<int64_t>(kDecodeMaxQuantizers, ceil_div(kblocks, QKB));
    p.bpq = (int)ceil_div(kblocks, p.nq);
    p.nq = (int)ceil_div(kblocks, p.bpq);                 // every quantizer owns k-blocks
    const int64_t streamers = std::max(1, sms - p.nq);
    const int64_t per_cta = ceil_div(N, streamers * DMMA_M);               // bands per CTA
    p.Rt = (int)std::min<int64_t>(DMMA_M, align_up(ceil_div(N, streamers * per_cta), 8));
    p.tiles = (int)ceil_div(N, p.Rt);
    p.grid = p.nq + (int)std::min<int64_t>(p.tiles, streamers);
    p.kblocks = (int)ceil_div(K, DBK);
    p.rows = image_rows((int)M);
    // shared memory of a streamer: [image ring (+ zero atom)][tail][xo][weight ring][slack for
    // the MMA's 128 rows]; the quantizer uses the first sizeof(QShared) bytes
    p.nst = (int)ceil_div(p.kblocks, DKS);
    const int64_t istage = (int64_t)DKS * p.rows * DBK;
    p.resident = p.nst <= DIMG_MAX && p.nst * istage <= DIMG_BYTES;
    p.nistage = p.resident ? p.nst : (int)std::min<int64_t>(DIMG_MAX, DIMG_BYTES / istage);
    const int64_t img = align_up((int64_t)p.nistage * istage + (p.rows == 8 ? 1024 : 0), 1024);
    p.tail_off = (uint32_t)img;
    p.xo_off = (uint32_t)align_up(p.tail_off + (int64_t)sizeof(DTail), 16);
    p.ring_off = (uint32_t)align_up(p.xo_off + std::max<int64_t>(cap, 1) * DM * 2, 1024);
    const int64_t stage = (int64_t)DKS * p.Rt * DBK;
    const int64_t slack = (int64_t)(DMMA_M - p.Rt) * DBK;
    const int64_t room = SMEM_LIMIT - 1024 - (int64_t)p.ring_off - slack;
    p.stages = (int)std::max<int64_t>(0, std::min<int64_t>(DMAX_STAGES, room / stage));
    p.inflight = std::max(1, std::min(DINFLIGHT, p.stages));
    // a quantizer: tables, its slice of X, the image of its k-blocks
    const int64_t qsmem = QX_OFF + M * p.bpq * DBK * 2 + (int64_t)p.bpq * p.rows * DBK + 1024;
    p.smem = (int)std::max<int64_t>(p.ring_off + p.stages * stage + slack + 1024, qsmem);
    return p;
}

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
    const DecodePlan p = decode_plan(d.M, d.N, d.K, d.cap, sms);
    if (p.stages < 2 || p.smem > SMEM_LIMIT || p.bpq * DBK / 8 > QMAX_CHUNKS)
        return cudaErrorInvalidValue;

    DArgs a;
    a.X = d.X;
    a.CB = d.CB;
    a.SCB = d.SCB;
    a.W16 = d.W16;
    a.bias = d.bias;
    a.Y = d.Y;
    a.C_debug = d.C_debug;
    a.Wo = d.Wo;
    a.wo_pitch = d.wo_pitch;
    a.bitmaps = d.bitmaps;
    a.n_bitmaps = (int)d.n_bitmaps;
    a.ybits = d.ybits;
    a.ytf = d.ybits && d.ythreshold > 0.0f ? fp16_rounded_threshold_f32(d.ythreshold) : 0.0f;
    a.ybits_all = d.ybits && d.ythreshold <= 0.0f ? 1 : 0;
    a.ncols32 = (int)(ceil_div(d.N, 32) * 32);
    a.count = d.count;
    a.table = d.table;
    a.image = d.image;
    a.status = d.status;
    a.epoch = d.status.tag >> 4;
    a.M = (int)d.M;
    a.N = (int)d.N;
    a.K = (int)d.K;
    a.cap = (int)d.cap;
    a.threshold = d.threshold;
    a.thr2 = fp16_threshold_pair(d.threshold);   // threshold > 0 on this path
    a.rows = p.rows;
    a.Rt = p.Rt;
    a.tiles = p.tiles;
    a.kblocks = p.kblocks;
    a.stages = p.stages;
    a.inflight = p.inflight;
    a.nq = p.nq;
    a.bpq = p.bpq;
    a.nst = p.nst;
    a.nistage = p.nistage;
    a.resident = p.resident ? 1 : 0;
    a.tail_off = p.tail_off;
    a.xo_off = p.xo_off;
    a.ring_off = p.ring_off;
    a.timeout_ns = d.timeout_ns;

    auto enc = encoder();
    if (!enc) return cudaErrorInvalidValue;
    CUtensorMap tm;
    cuuint64_t dims[2] = {(cuuint64_t)d.K, (cuuint64_t)d.N};
    cuuint64_t strides[1] = {(cuuint64_t)d.K};
    cuuint32_t box[2] = {DBK, (cuuint32_t)p.Rt};
    cuuint32_t estr[2] = {1, 1};
    if (enc(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<int8_t *>(d.CB), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;

    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.gridDim = dim3((unsigned)p.grid);
    cfg.blockDim = dim3(DTHREADS);
    cfg.dynamicSmemBytes = (size_t)p.smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    err = cudaLaunchKernelEx(&cfg, llmint8_decode_kernel, tm, a);
    note_launches(1);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace llmint8

// Device-side building blocks shared by the sm_100a kernels of the LLM.int8() layer:
// mbarrier / TMA / tcgen05 wrappers (inline PTX) and the bounded wait used by every
// pipeline loop.  Nothing here allocates memory.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "llmint8.h"

namespace llmint8 {

// Layout of the first 256 bytes of every workspace.
struct WsHeader {
    unsigned long long status;   // (call epoch << 4) | llmint8_status, one writer per call
    unsigned long long timeout;  // (call epoch << 4) | LLMINT8_ERR_TIMEOUT after a timeout (or,
                                 // debug build, | LLMINT8_ERR_DEVICE_CHECK after a failed check)
    int32_t n_outliers;          // true number of outlier columns found by the last call
    uint32_t pad[59];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

__host__ __device__ constexpr int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }
__host__ __device__ constexpr int64_t ceil_div(int64_t x, int64_t a) { return (x + a - 1) / a; }

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ------------------------------------------------------------------ mbarrier ----------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Device-side conditions of a call.  Every call gets a new epoch.  Exactly one thread of
// the call stores (epoch << 4) | code into the status word (the outlier-count result,
// written before anything can time out in that kernel); any thread whose bounded wait
// gives up stores (epoch << 4) | TIMEOUT into the timeout word, and in the debug build any
// thread whose device check fails stores (epoch << 4) | DEVICE_CHECK there.  The host
// reports the timeout word's code when both words carry the same epoch, else the status
// word's code.  Plain stores of one value per word: no ordering between CTAs or kernels
// matters and the workspace needs no initialization.
struct StatusRef {
    unsigned long long *word;
    unsigned long long *timeout_word;
    unsigned long long tag;     // epoch << 4
    __device__ __forceinline__ void set(llmint8_status code) const {
        *reinterpret_cast<volatile unsigned long long *>(word) = tag | (unsigned long long)code;
    }
    __device__ __forceinline__ void timed_out() const {
        *reinterpret_cast<volatile unsigned long long *>(timeout_word) =
            tag | (unsigned long long)LLMINT8_ERR_TIMEOUT;
    }
    __device__ __forceinline__ void check_failed() const {
        *reinterpret_cast<volatile unsigned long long *>(timeout_word) =
            tag | (unsigned long long)LLMINT8_ERR_DEVICE_CHECK;
    }
};

// Packed-half helpers on raw bits: |x| (clear the sign bits), |x| >= t per half (0xffff
// where true), max per half.  fp16 comparisons and maxima are exact.
__device__ __forceinline__ uint32_t habs2_bits(uint32_t v) { return v & 0x7fff7fffu; }
__device__ __forceinline__ uint32_t hge2_bits(uint32_t a, uint32_t t) {
    return __hge2_mask(*reinterpret_cast<const __half2 *>(&a), *reinterpret_cast<const __half2 *>(&t));
}
__device__ __forceinline__ uint32_t hmax2_bits(uint32_t a, uint32_t b) {
    const __half2 r = __hmax2(*reinterpret_cast<const __half2 *>(&a),
                              *reinterpret_cast<const __half2 *>(&b));
    return *reinterpret_cast<const uint32_t *>(&r);
}

// A threshold t as the smallest fp16 >= t, in both halves of a word: for an fp16 x,
// |x| >= t exactly when |x| >= that value (fp16 compares, packed two at a time), for every t
// (zero, negative and past the fp16 range included; a NaN x compares false either way).
inline uint32_t fp16_threshold_pair(float t) {
    const __half t16 = __float2half_ru(t);
    const uint32_t tb = (uint32_t)*reinterpret_cast<const uint16_t *>(&t16);
    return tb | (tb << 16);
}

// For a threshold t > 0: the smallest fp32 f >= 0 with |fp16_rn(f)| >= (the smallest fp16
// >= t), so that for every fp32 y, |fp16_rn(y)| >= t exactly when |y| >= f (fp16 rounding to
// nearest is monotone).  Found by bisection over the non-negative fp32 bit patterns.
inline float fp16_rounded_threshold_f32(float t) {
    const float t16 = __half2float(__float2half_ru(t));   // may be +inf
    uint32_t lo = 0u, hi = 0x7f800000u;                     // f(hi) = +inf qualifies
    while (lo < hi) {
        const uint32_t mid = lo + (hi - lo) / 2;
        float f;
        memcpy(&f, &mid, 4);
        if (__half2float(__float2half_rn(f)) >= t16) hi = mid;
        else lo = mid + 1;
    }
    float f;
    memcpy(&f, &lo, 4);
    return f;
}

// Device-side bounds check of the debug build (compiled with LLMINT8_DEBUG): a false
// condition records LLMINT8_ERR_DEVICE_CHECK through `status` and execution goes on.  The
// release build compiles it to nothing.
#ifdef LLMINT8_DEBUG
#define LLMINT8_DCHECK(cond, status)          \
    do {                                      \
        if (!(cond)) (status).check_failed(); \
    } while (0)
#else
#define LLMINT8_DCHECK(cond, status) \
    do {                             \
    } while (0)
#endif

// Every wait of a pipeline goes through this: it gives up after `timeout_ns`, or as soon
// as another thread of the CTA gave up, records LLMINT8_ERR_TIMEOUT in the workspace
// status word and returns false so that the caller can wind the kernel down.
struct BoundedWait {
    volatile int *abort_flag;   // shared memory, one per CTA
    StatusRef status;
    uint64_t timeout_ns;

    __device__ __forceinline__ bool operator()(uint32_t bar, uint32_t parity) const {
        if (mbar_try_wait(bar, parity)) return true;
        const uint64_t t0 = global_timer_ns();
        for (uint32_t it = 1;; ++it) {
            if (mbar_try_wait(bar, parity)) return true;
            if ((it & 63u) == 0u) {
                if (*abort_flag) return false;
                if (global_timer_ns() - t0 > timeout_ns) {
                    *abort_flag = 1;
                    status.timed_out();
                    return false;
                }
            }
        }
    }
};

// Wait used while winding down (draining copies / MMAs still in flight): ignores the abort
// flag, bounded by a fixed limit.
__device__ __forceinline__ bool drain_wait(uint32_t bar, uint32_t parity, StatusRef status) {
    constexpr uint64_t kDrainNs = 1000000000ull;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 63u) == 0u && global_timer_ns() - t0 > kDrainNs) {
            status.timed_out();
            return false;
        }
    }
}

// ---------------------------------------------------------------------- TMA -----------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *tm) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm)) : "memory");
}
// 2-D tiled bulk load global -> shared, completion counted on `bar` in bytes.
// x (innermost coordinate) is always a multiple of 16 bytes here.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *tm, int x, int y,
                                            uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}

// Contiguous bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16),
// completion counted on `bar` in bytes.
__device__ __forceinline__ void bulk_load_1d(uint32_t dst, const void *src, uint32_t bytes,
                                             uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}

// ------------------------------------------------------------ thread-block clusters -----
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory variable in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
__device__ __forceinline__ void st_cluster_u8(uint32_t addr, uint32_t v) {
    asm volatile("st.shared::cluster.u8 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}
// Arrive (release, cluster scope) on an mbarrier of another CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t remote_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(remote_bar)
                 : "memory");
}
// Hardware barrier over every thread of every CTA of the cluster (used once, right after
// the mbarriers are initialized, before any CTA may arrive on a peer's mbarrier).
__device__ __forceinline__ void cluster_barrier_all() {
    asm volatile(
        "barrier.cluster.arrive.release.aligned;\n\t"
        "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Asks L2 to fetch one box of a tensor map (no shared memory, nothing to wait for).
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *tm, int x, int y) {
    asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global [%0, {%1, %2}];" ::"l"(
                     reinterpret_cast<uint64_t>(tm)),
                 "r"(x), "r"(y)
                 : "memory");
}

// ------------------------------------------------------------------- tcgen05 ----------
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Warp-wide: allocate `ncols` TMEM columns, address written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, both K-major; int8 x int8 -> int32.
__device__ __forceinline__ void mma_i8(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// D[tmem] (+)= A[smem] * B[smem]^T, both K-major; f16 x f16 -> f32.
__device__ __forceinline__ void mma_f16(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
        : "memory");
}
// Warp-wide: 32 lanes x 32 consecutive 32-bit columns from TMEM into registers.
__device__ __forceinline__ void tmem_ld_32x32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}
// Warp-wide: 32 lanes x 16 consecutive 32-bit columns from TMEM into registers.
__device__ __forceinline__ void tmem_ld_32x16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
// Orders this thread's generic-proxy global accesses with later async-proxy ones (bulk
// copies / TMA) - in the same thread, and, after a release/acquire, across threads.
__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}
// Named barrier over `count` threads (a multiple of 32).
__device__ __forceinline__ void named_barrier(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor of a K-major tile written by TMA with 128-byte swizzle:
// rows of 128 bytes, 8-row groups 1024 bytes apart (tile base 1024-byte aligned).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);      // start address / 16
    d |= (uint64_t)1u << 16;                      // leading byte offset (unused, 16 B)
    d |= (uint64_t)(1024u >> 4) << 32;            // stride byte offset: 8 rows * 128 B
    d |= (uint64_t)1u << 46;                      // descriptor version (sm_100)
    d |= (uint64_t)2u << 61;                      // swizzle: 128 B
    return d;
}

// Order in which a tile walks its k-blocks: rotated by a tile-dependent offset, so that the
// CTAs streaming different tiles at the same moment read different column ranges of the
// 2^n-strided weight rows (spreading the requests over the DRAM channels) instead of all
// hitting the same offset.  Integer accumulation makes the order irrelevant to the result.
__host__ __device__ __forceinline__ int rotated_kblock(int it, int tile, int kblocks) {
    const int r = (int)(((unsigned)tile * 7u) % (unsigned)kblocks);
    const int kb = it + r;
    return kb >= kblocks ? kb - kblocks : kb;
}

// Instruction descriptors (kind::i8 and kind::f16), K-major A and B, dense.
//   bits 4-5 accumulator type (1 = f32, 2 = s32); 7-9 A type; 10-12 B type
//   (i8: 1 = signed; f16: 0 = fp16); 17-22 N/8; 24-28 M/16.
__host__ __device__ constexpr uint32_t idesc_i8(int m, int n) {
    return (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) |
           ((uint32_t)(m >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_f16(int m, int n) {
    return (1u << 4) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

}  // namespace llmint8

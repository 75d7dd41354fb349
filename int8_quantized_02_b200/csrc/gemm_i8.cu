// The LLM.int8() product on the 5th-generation tensor cores of sm_100a.
//
// One persistent CTA per SM computes 128 x 256 output tiles (or, for M > 128, a pair of CTAs in
// a cluster computes 256 x 256 tiles with tcgen05.mma.cta_group::2: each CTA holds its 128
// rows of Xq and 128 of the 256 weight rows of a stage, and its TMEM the 128 x 256 result of
// its rows; the pair halves the weight bytes each SM brings in per MAC and fits six stages)
// of
//     Y = fp16( C * SCA_i * SCB_n / 127^2 + P + bias_n ),
//     C = Xq . CB^T    (int8 x int8 -> int32, tcgen05.mma kind::i8, exact)
//     P = Xo . Wo^T    (fp16 x fp16 -> fp32, tcgen05.mma kind::f16, the outlier columns)
// which is the decomposition of the LLM.int8() summary (sections الابتكار الثاني and
// الصورة الكاملة) and of the blog's three steps (section LLM.int8() 温和总结): the regular part
// goes through the int8 product dequantized by the outer product of the row and column
// absmax vectors, the outlier part through a 16-bit product, and the two are summed in the
// epilogue before the single rounding to fp16.
//
// Warp roles (320 threads):
//   warp 0      TMA producer: k-blocks of Xq / CB (128 B of K each), then of Xo / Wo
//               (64 fp16 of K each) - both fill the same shared-memory stages (48 KB, or
//               32 KB per CTA of a pair, whose loads complete on the pair leader's barrier);
//   warp 1      TMEM allocator and MMA issuer (one thread; of a pair, the leader's only);
//   warps 2..9  epilogue: TMEM -> registers -> dequantize, add P and bias -> fp16 -> global;
//               warp w reads TMEM lanes 32 * (w % 4) (the hardware's lane quadrant), and the
//               two warps of a quadrant take the two halves of the tile's columns.
// TMEM (512 columns): the int32 accumulator is double-buffered (2 x 256 columns) so the
// epilogue of a tile overlaps the main loop of the next.  The outlier product P takes one of
// two routes:
//   few outlier columns (n_out <= kRegOutliers, the usual case: a handful of feature
//   dimensions) - the epilogue warps form P on the CUDA cores (fp32 FMAs) from their rows of
//   Xo and the tile's slice of Wo, both staged in shared memory while the main loop of the
//   tile runs;
//   more - P is a tcgen05 kind::f16 product appended to the k-loop, accumulated in fp32 in
//   the second half of TMEM, and the int32 accumulator is single-buffered.
// Every wait is bounded (BoundedWait); a timeout records LLMINT8_ERR_TIMEOUT, drains the
// copies and MMAs in flight, frees TMEM and returns.  A pair's CTAs exit only after the
// leader has drained the loads of both and the second CTA has made its last arrive on the
// leader's barriers.
#include <cudaTypedefs.h>

#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace llmint8 {

namespace {

constexpr int BM = 128;                 // tile rows (M) held by one CTA
constexpr int BN = 256;                 // tile columns (N)
constexpr int BKB = 128;                // bytes of K per stage row (128 int8 or 64 fp16)
// Epilogue warps: two per TMEM lane quadrant, each taking half of the tile's columns, so
// that two warps per scheduler share the epilogue work of a tile.
constexpr int EPI_WARPS = 8;
constexpr int THREADS = 64 + 32 * EPI_WARPS;

// Single CTA (PAIR = false): 128 x 256 tiles, 4 stages of 16 + 32 KB.  CTA pair: 256 x 256
// tiles, each CTA 6 stages of 16 KB (its Xq rows) + 16 KB (its half of the weight rows).
template <bool PAIR>
struct Cfg {
    static constexpr int STAGES = PAIR ? 6 : 4;
    static constexpr int B_ROWS = PAIR ? BN / 2 : BN;
    static constexpr int TILE_M = PAIR ? 2 * BM : BM;
    static constexpr int A_BYTES = BM * BKB;
    static constexpr int B_BYTES = B_ROWS * BKB;
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
};
constexpr uint32_t TMEM_COLS = 512;
constexpr int kRegOutliers = 16;        // outlier columns formed in the epilogue at most
// the tile's column slice, staged once per tile by the four epilogue warps together:
// Wo [o][n] fp16, SCB [n] and bias [n] as fp32; and per epilogue warp its rows of Xo,
// [o][lane] fp32
constexpr int SL_W_BYTES = kRegOutliers * BN * 2;
constexpr int SL_XO_WARP = kRegOutliers * 32 * 4;
constexpr int SL_BYTES = SL_W_BYTES + BN * 4 + BN * 4 + EPI_WARPS * SL_XO_WARP;

template <int NSTAGES>
struct Tail {
    uint64_t full[NSTAGES];
    uint64_t empty[NSTAGES];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t mma_done;
    uint64_t slice_full;                // the epilogue warps staged the column slice
    uint64_t slice_empty;               // ... and are done reading it
    uint64_t loads_drained;             // pair, second CTA: the leader drained every load
    uint64_t peer_exit;                 // pair, leader: the second CTA made its last arrive
    uint32_t tmem_base;
    int abort_flag;
};
template <bool PAIR>
constexpr int smem_bytes() {
    return Cfg<PAIR>::STAGES * Cfg<PAIR>::STAGE_BYTES + SL_BYTES + 1024 +
           (int)sizeof(Tail<Cfg<PAIR>::STAGES>);
}
static_assert(smem_bytes<false>() <= 232448, "fits the opt-in shared memory of one CTA");
static_assert(smem_bytes<true>() <= 232448, "fits the opt-in shared memory of one CTA");

struct Args {
    const __half *Xo;        // [M, pitch]
    const __half *Wo;        // [N, pitch]
    int pitch;
    const int32_t *count;
    int64_t cap;
    const float *SCA;
    const float *SCB;
    const __half *bias;
    __half *Y;
    int32_t *C_debug;
    uint32_t *ybits;         // outlier bitmaps of Y for the next layer, or null
    int ybits_words;         // ceil(N / 32)
    float ytf;               // its threshold on the fp32 value (fp16_rounded_threshold_f32)
    int ybits_all;           // threshold <= 0: every column
    StatusRef status;
    int M, N, K;
    int num_kb;
    int tiles_m, tiles_n;
    uint64_t timeout_ns;
};

// ---- CTA-pair forms (tcgen05 cta_group::2).  The pair's leader (rank 0) issues the MMAs;
// operand addresses are the same shared-memory offsets in both CTAs.
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap *tm, int x,
                                                 int y, uint32_t bar_cluster) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_cluster)
        : "memory");
}
// The same loads with an L2 eviction policy.  The quantized rows Xq are re-read by every wave
// of output tiles (the tiles walk M fastest), so their loads ask L2 to evict them last; the
// weight loads keep the default policy (the 16 M tiles of a weight tile do not all run at the
// same moment, and evict-first weights were re-read from HBM: 2.78 against 1.72 GB per
// launch on the 175B projection, while evict-last Xq alone gives 1.55 GB).
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ void tma_load_2d_hint(uint32_t dst, const CUtensorMap *tm, int x, int y,
                                                 uint32_t bar, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void tma_load_2d_pair_hint(uint32_t dst, const CUtensorMap *tm, int x,
                                                      int y, uint32_t bar_cluster, uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(tm)), "r"(x), "r"(y), "r"(bar_cluster), "l"(pol)
        : "memory");
}
__device__ __forceinline__ void mma_i8_pair(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void mma_f16_pair(uint32_t d, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
// Arrive on the barrier at `bar` in both CTAs of the pair once the pair's MMAs issued so far
// by this thread have completed: one commit for each CTA's barrier (a commit tracks every
// earlier tcgen05 operation of the thread, so the two arrive at the same point).
__device__ __forceinline__ void tc_commit_pair_both(uint32_t bar) {
#pragma unroll
    for (uint32_t r = 0; r < 2; ++r)
        asm volatile(
            "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                map_to_rank(bar, r))
            : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_half2(float a, float b) {
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t *>(&h);
}

template <bool PAIR, bool YBITS>
__device__ __forceinline__ void gemm_body(const CUtensorMap &tmA, const CUtensorMap &tmB,
                                          const CUtensorMap &tmXo, const CUtensorMap &tmWo,
                                          const Args &a) {
    using C = Cfg<PAIR>;
    constexpr int STAGES = C::STAGES;
    constexpr int STAGE_BYTES = C::STAGE_BYTES;
    constexpr int A_BYTES = C::A_BYTES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __half *sl_w = reinterpret_cast<__half *>(smem + STAGES * STAGE_BYTES);
    float *sl_scb = reinterpret_cast<float *>(smem + STAGES * STAGE_BYTES + SL_W_BYTES);
    float *sl_bias = sl_scb + BN;
    float *sl_xo = sl_bias + BN;
    Tail<STAGES> *tail = reinterpret_cast<Tail<STAGES> *>(smem + STAGES * STAGE_BYTES + SL_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // the pair: rank 0 is the leader; tiles are numbered per pair
    const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
    const bool leader = rank == 0;
    const int unit = PAIR ? (int)(blockIdx.x >> 1) : (int)blockIdx.x;
    const int units = PAIR ? (int)(gridDim.x >> 1) : (int)gridDim.x;

    // Prologue: nothing here reads global memory that the kernels before this one write, so
    // it overlaps their tail (this grid is their programmatic dependent).
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_addr(&tail->full[s]), 1);
            mbar_init(smem_addr(&tail->empty[s]), 1);
        }
        for (int s = 0; s < 2; ++s) {
            mbar_init(smem_addr(&tail->acc_full[s]), 1);
            // the epilogue warps of this CTA (and of the second CTA of a pair) release it
            mbar_init(smem_addr(&tail->acc_empty[s]), PAIR ? 2 * EPI_WARPS : EPI_WARPS);
        }
        mbar_init(smem_addr(&tail->mma_done), 1);
        mbar_init(smem_addr(&tail->slice_full), EPI_WARPS);
        mbar_init(smem_addr(&tail->slice_empty), EPI_WARPS);
        mbar_init(smem_addr(&tail->loads_drained), 1);
        mbar_init(smem_addr(&tail->peer_exit), 1);
        tail->abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        if (a.cap > 0) {
            tma_prefetch_desc(&tmXo);
            tma_prefetch_desc(&tmWo);
        }
    }
    if (warp == 1) {
        if (PAIR) tmem_alloc_pair(smem_addr(&tail->tmem_base), TMEM_COLS);
        else tmem_alloc(smem_addr(&tail->tmem_base), TMEM_COLS);
    }
    // a pair's barriers are initialized in both CTAs before either may use the other's
    if (PAIR) cluster_barrier_all();
    // the quantized operands, scales and outlier list of this call are complete after this
    asm volatile("griddepcontrol.wait;" ::: "memory");
    // No early launch_dependents: the kernel after this one (the next call's outlier scan)
    // then starts when this grid ends instead of parking its CTAs beside the GEMM's; with
    // eight epilogue warps that was 6 % faster on the 6.7B FFN step.

    // Outlier configuration of this call (uniform over the grid).
    const int n_out = (int)min((int64_t)*a.count, a.cap);
    LLMINT8_DCHECK(n_out >= 0 && n_out <= a.cap && n_out <= a.K, a.status);
    const bool all_outliers = n_out >= a.K;            // then C == 0: skip the int8 blocks
    const bool reg_out = n_out > 0 && n_out <= kRegOutliers && !all_outliers;
    const int nob = reg_out ? 0 : (n_out + 63) / 64;   // fp16 k-blocks of 64 columns
    const int nkb = all_outliers ? 0 : a.num_kb;
    const int acc_stages = nob > 0 ? 1 : 2;
    const int total_tiles = a.tiles_m * a.tiles_n;

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const BoundedWait wait{&tail->abort_flag, a.status, a.timeout_ns};

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer ----
        if (lane == 0) {
            const uint64_t keep = l2_policy_evict_last();
            int stage = 0;
            uint32_t phase = 0;
            uint32_t used = 0, last_parity = 0;   // per stage: issued at least once / parity
            for (int tile = unit; tile < total_tiles; tile += units) {
                // this CTA's rows of X and of the weight tile
                const int m0 = (tile % a.tiles_m) * C::TILE_M + (int)rank * BM;
                const int n0 = (tile / a.tiles_m) * BN + (int)rank * C::B_ROWS;
                for (int kb = 0; kb < nkb + nob; ++kb) {
                    if (!wait(smem_addr(&tail->empty[stage]), phase ^ 1)) goto drain;
                    const uint32_t full = smem_addr(&tail->full[stage]);
                    const uint32_t sa = smem_addr(smem + stage * STAGE_BYTES);
                    if (!PAIR || leader)   // the leader's barrier counts the bytes of both CTAs
                        mbar_arrive_expect_tx(full, PAIR ? 2 * STAGE_BYTES : STAGE_BYTES);
                    const uint32_t fbar = PAIR ? map_to_rank(full, 0) : full;
                    if (kb < nkb) {
                        const int kr = rotated_kblock(kb, tile / a.tiles_m, nkb);
                        if (PAIR) {
                            tma_load_2d_pair_hint(sa, &tmA, kr * BKB, m0, fbar, keep);
                            tma_load_2d_pair(sa + A_BYTES, &tmB, kr * BKB, n0, fbar);
                        } else {
                            tma_load_2d_hint(sa, &tmA, kr * BKB, m0, full, keep);
                            tma_load_2d(sa + A_BYTES, &tmB, kr * BKB, n0, full);
                        }
                    } else {
                        const int x = (kb - nkb) * (BKB / 2);
                        if (PAIR) {
                            tma_load_2d_pair(sa, &tmXo, x, m0, fbar);
                            tma_load_2d_pair(sa + A_BYTES, &tmWo, x, n0, fbar);
                        } else {
                            tma_load_2d(sa, &tmXo, x, m0, full);
                            tma_load_2d(sa + A_BYTES, &tmWo, x, n0, full);
                        }
                    }
                    used |= 1u << stage;
                    last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
            }
        drain:
            // wait for every copy this thread issued to land before the CTA may exit (a pair's
            // leader waits for the copies of both CTAs, then tells the second CTA)
            if (!PAIR || leader) {
                for (int s = 0; s < STAGES; ++s)
                    if (used & (1u << s))
                        drain_wait(smem_addr(&tail->full[s]), (last_parity >> s) & 1u, a.status);
                if (PAIR) mbar_arrive_cluster(map_to_rank(smem_addr(&tail->loads_drained), 1));
            }
        }
    } else if (warp == 1) {
        // --------------------------------------------------------------- MMA issuer ----
        if (lane == 0 && (!PAIR || leader)) {
            const uint32_t id_i8 = idesc_i8(C::TILE_M, BN);
            const uint32_t id_f16 = idesc_f16(C::TILE_M, BN);
            int stage = 0;
            uint32_t phase = 0;
            int acc = 0;
            uint32_t acc_phase = 0;
            for (int tile = unit; tile < total_tiles; tile += units) {
                if (!wait(smem_addr(&tail->acc_empty[acc]), acc_phase ^ 1)) break;
                tc_fence_after();
                const uint32_t d_i32 = tmem + (uint32_t)(acc * 256);
                const uint32_t d_f32 = tmem + 256u;
                bool ok = true;
                for (int kb = 0; kb < nkb + nob; ++kb) {
                    if (!wait(smem_addr(&tail->full[stage]), phase)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = smem_addr(smem + stage * STAGE_BYTES);
                    const uint32_t sb = sa + A_BYTES;
                    if (kb < nkb) {
#pragma unroll
                        for (int k = 0; k < BKB / 32; ++k) {
                            if (PAIR)
                                mma_i8_pair(d_i32, sw128_desc(sa + 32 * k),
                                            sw128_desc(sb + 32 * k), id_i8, (kb | k) != 0);
                            else
                                mma_i8(d_i32, sw128_desc(sa + 32 * k), sw128_desc(sb + 32 * k),
                                       id_i8, (kb | k) != 0);
                        }
                    } else {
#pragma unroll
                        for (int k = 0; k < BKB / 32; ++k) {
                            if (PAIR)
                                mma_f16_pair(d_f32, sw128_desc(sa + 32 * k),
                                             sw128_desc(sb + 32 * k), id_f16,
                                             ((kb - nkb) | k) != 0);
                            else
                                mma_f16(d_f32, sw128_desc(sa + 32 * k), sw128_desc(sb + 32 * k),
                                        id_f16, ((kb - nkb) | k) != 0);
                        }
                    }
                    // frees the stage (in both CTAs of a pair)
                    if (PAIR) tc_commit_pair_both(smem_addr(&tail->empty[stage]));
                    else tc_commit(smem_addr(&tail->empty[stage]));
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1;
                    }
                }
                if (!ok) break;
                // accumulators ready (in both CTAs of a pair)
                if (PAIR) tc_commit_pair_both(smem_addr(&tail->acc_full[acc]));
                else tc_commit(smem_addr(&tail->acc_full[acc]));
                if (++acc == acc_stages) {
                    acc = 0;
                    acc_phase ^= 1;
                }
            }
            // every MMA issued by this thread has completed once mma_done arrives
            if (PAIR) tc_commit_pair_both(smem_addr(&tail->mma_done));
            else tc_commit(smem_addr(&tail->mma_done));
            drain_wait(smem_addr(&tail->mma_done), 0, a.status);
        } else if (lane == 0) {
            // second CTA of a pair: its TMEM and shared memory are the leader's MMA operands
            // until the leader's last MMA has completed
            drain_wait(smem_addr(&tail->mma_done), 0, a.status);
        }
    } else {
        // ----------------------------------------------------------------- epilogue ----
        const int q = warp & 3;                        // TMEM lane quadrant of this warp
        const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
        const int wq = warp - 2;                       // this warp's share of the slice
        constexpr int kSliceCols = BN / EPI_WARPS;      // columns it stages
        constexpr int kChunks = BN / 32 / (EPI_WARPS / 4);   // 32-column chunks it finishes
        const int c0 = (wq / 4) * kChunks;              // its first chunk
        int acc = 0;
        uint32_t acc_phase = 0, sl_phase = 0;
        bool first = true;
        for (int tile = unit; tile < total_tiles; tile += units) {
            const int m0 = (tile % a.tiles_m) * C::TILE_M + (int)rank * BM;   // this CTA's rows
            const int n0 = (tile / a.tiles_m) * BN;
            // The tile's column slice (SCB, bias and, with few outlier columns, Wo), staged
            // while the tensor cores still work on the tile: each warp an equal share of it,
            // after every warp is done with the previous tile's slice.
            {
                int okq = 1;
                if (lane == 0 && !first)
                    okq = wait(smem_addr(&tail->slice_empty), sl_phase ^ 1) ? 1 : 0;
                okq = __shfl_sync(0xffffffffu, okq, 0);
                if (!okq) break;
                for (int cc = wq * kSliceCols + lane; cc < (wq + 1) * kSliceCols; cc += 32) {
                    const int n = n0 + cc;
                    const bool in = n < a.N;
                    sl_scb[cc] = in ? __ldg(a.SCB + n) : 0.0f;
                    sl_bias[cc] = (in && a.bias) ? __half2float(a.bias[n]) : 0.0f;
                    if (reg_out) {
#pragma unroll
                        for (int o8 = 0; o8 < kRegOutliers; o8 += 8) {
                            if (o8 < n_out) {
                                uint4 v = make_uint4(0, 0, 0, 0);
                                if (in)
                                    v = __ldg(reinterpret_cast<const uint4 *>(
                                        a.Wo + (int64_t)n * a.pitch + o8));
                                const __half *h = reinterpret_cast<const __half *>(&v);
#pragma unroll
                                for (int e = 0; e < 8; ++e)
                                    if (o8 + e < n_out) sl_w[(o8 + e) * BN + cc] = h[e];
                            }
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&tail->slice_full));
                int okf = 0;
                if (lane == 0) okf = wait(smem_addr(&tail->slice_full), sl_phase) ? 1 : 0;
                okf = __shfl_sync(0xffffffffu, okf, 0);
                if (!okf) break;
                first = false;
            }
            // this thread's row of Xo (the outlier columns of X), [o][lane] in this warp's part
            float *xo_s = sl_xo + wq * (kRegOutliers * 32);
            if (reg_out) {
                const int r = m0 + q * 32 + lane;
                for (int o8 = 0; o8 < n_out; o8 += 8) {
                    uint4 v = make_uint4(0, 0, 0, 0);
                    if (r < a.M)
                        v = __ldg(reinterpret_cast<const uint4 *>(a.Xo + (int64_t)r * a.pitch + o8));
                    const __half *h = reinterpret_cast<const __half *>(&v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) xo_s[(o8 + e) * 32 + lane] = __half2float(h[e]);
                }
            }
            const int row = m0 + q * 32 + lane;
            const bool row_ok = row < a.M;
            const float rs = row_ok ? a.SCA[row] * (1.0f / 16129.0f) : 0.0f;
            int ok = 0;
            if (lane == 0) ok = wait(smem_addr(&tail->acc_full[acc]), acc_phase) ? 1 : 0;
            ok = __shfl_sync(0xffffffffu, ok, 0);
            if (!ok) break;
            tc_fence_after();
            for (int c = c0; c < c0 + kChunks; ++c) {
                const int nb = n0 + c * 32;
                if (nb >= a.N) break;
                uint32_t ci[32], pf[32];
                if (nkb > 0) tmem_ld_32x32(tl + (uint32_t)(acc * 256 + c * 32), ci);
                if (nob > 0) tmem_ld_32x32(tl + (uint32_t)(256 + c * 32), pf);
                tmem_wait_ld();
                if (nkb == 0) {
#pragma unroll
                    for (int j = 0; j < 32; ++j) ci[j] = 0u;
                }
                if (nob == 0) {
                    float p[32];
#pragma unroll
                    for (int j = 0; j < 32; ++j) p[j] = 0.0f;
                    if (reg_out) {
                        // P[row, nb + j] = sum_o Xo[row, o] * Wo[nb + j, o], o ascending
#pragma unroll 1
                        for (int o = 0; o < n_out; ++o) {
                            const float xv = xo_s[o * 32 + lane];
                            const uint4 *wv = reinterpret_cast<const uint4 *>(sl_w + o * BN + c * 32);
#pragma unroll
                            for (int v = 0; v < 4; ++v) {
                                const uint4 w8 = wv[v];
                                const __half2 *h = reinterpret_cast<const __half2 *>(&w8);
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const float2 wf = __half22float2(h[e]);
                                    p[v * 8 + 2 * e] = fmaf(xv, wf.x, p[v * 8 + 2 * e]);
                                    p[v * 8 + 2 * e + 1] = fmaf(xv, wf.y, p[v * 8 + 2 * e + 1]);
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) pf[j] = __float_as_uint(p[j]);
                }
                const int groups = min(32, a.N - nb) / 16;   // 1 or 2 groups of 16 columns
                uint32_t ymask = 0;   // bit j: |fp16 Y[row, nb + j]| >= the next threshold
                if (row_ok) {
                    __half *yrow = a.Y + (int64_t)row * a.N + nb;
                    int32_t *crow = a.C_debug ? a.C_debug + (int64_t)row * a.N + nb : nullptr;
#pragma unroll
                    for (int g = 0; g < 2; ++g) {
                        if (g < groups) {
                            uint32_t packed[8];
#pragma unroll
                            for (int j4 = 0; j4 < 4; ++j4) {
                                const int cj = c * 32 + g * 16 + j4 * 4;
                                const float4 sb = *reinterpret_cast<const float4 *>(sl_scb + cj);
                                const float4 bv = *reinterpret_cast<const float4 *>(sl_bias + cj);
                                const float b[4] = {bv.x, bv.y, bv.z, bv.w};
                                const float sbv[4] = {sb.x, sb.y, sb.z, sb.w};
                                float y[4];
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int j = g * 16 + j4 * 4 + e;
                                    y[e] = fmaf((float)(int32_t)ci[j], rs * sbv[e],
                                                __uint_as_float(pf[j]) + b[e]);
                                }
                                if (YBITS) {
                                    // |fp16(y)| >= the next threshold <=> |y| >= ytf
#pragma unroll
                                    for (int e = 0; e < 4; ++e)
                                        ymask |= (fabsf(y[e]) >= a.ytf ? 1u : 0u)
                                                 << (g * 16 + j4 * 4 + e);
                                }
                                packed[j4 * 2] = pack_half2(y[0], y[1]);
                                packed[j4 * 2 + 1] = pack_half2(y[2], y[3]);
                            }
                            LLMINT8_DCHECK(row < a.M && nb + g * 16 + 16 <= a.N, a.status);
                            uint4 *dst = reinterpret_cast<uint4 *>(yrow + g * 16);
                            dst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
                            dst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
                            if (crow) {
                                uint4 *cd = reinterpret_cast<uint4 *>(crow + g * 16);
#pragma unroll
                                for (int v = 0; v < 4; ++v)
                                    cd[v] = make_uint4(ci[g * 16 + v * 4], ci[g * 16 + v * 4 + 1],
                                                       ci[g * 16 + v * 4 + 2],
                                                       ci[g * 16 + v * 4 + 3]);
                            }
                        }
                    }
                }
                if (YBITS) {
                    // OR over the warp's 32 rows: one word of this 32-row block's bitmap
                    if (a.ybits_all && row_ok) ymask = groups == 2 ? 0xffffffffu : 0xffffu;
                    const uint32_t word = __reduce_or_sync(0xffffffffu, ymask);
                    if (lane == 0 && m0 + q * 32 < a.M) {
                        LLMINT8_DCHECK(nb < a.N, a.status);
                        a.ybits[(int64_t)((m0 + q * 32) >> 5) * a.ybits_words + (nb >> 5)] = word;
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                // the accumulator buffer is free again (the leader's barrier for a pair)
                if (PAIR && !leader)
                    mbar_arrive_cluster(map_to_rank(smem_addr(&tail->acc_empty[acc]), 0));
                else
                    mbar_arrive(smem_addr(&tail->acc_empty[acc]));
                mbar_arrive(smem_addr(&tail->slice_empty));
            }
            sl_phase ^= 1;
            if (++acc == acc_stages) {
                acc = 0;
                acc_phase ^= 1;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (PAIR && threadIdx.x == 0) {
        if (leader) {
            // the second CTA has made its last arrive on this CTA's barriers
            drain_wait(smem_addr(&tail->peer_exit), 0, a.status);
        } else {
            // the leader has seen every copy of this CTA land; then release the leader
            drain_wait(smem_addr(&tail->loads_drained), 0, a.status);
            mbar_arrive_cluster(map_to_rank(smem_addr(&tail->peer_exit), 0));
        }
    }
    if (warp == 1) {
        tc_fence_after();
        if (PAIR) tmem_dealloc_pair(tmem, TMEM_COLS);
        else tmem_dealloc(tmem, TMEM_COLS);
    }
}

// The kernels: single CTAs (M <= 128) or clusters of two CTAs with 256 x 256 tiles (M > 128),
// each also in a form that writes the next layer's outlier bitmaps of Y (llmint8_linear_next_
// bitmaps), so that the plain form carries none of that work.
#define LLMINT8_GEMM_KERNEL(NAME, PAIR, YBITS)                                                   \
    __global__ void __launch_bounds__(THREADS, 1)                                               \
        NAME(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,  \
             const __grid_constant__ CUtensorMap tmXo, const __grid_constant__ CUtensorMap tmWo, \
             const Args a) {                                                                    \
        gemm_body<PAIR, YBITS>(tmA, tmB, tmXo, tmWo, a);                                        \
    }
LLMINT8_GEMM_KERNEL(llmint8_gemm_kernel, false, false)
LLMINT8_GEMM_KERNEL(llmint8_gemm_pair_kernel, true, false)
LLMINT8_GEMM_KERNEL(llmint8_gemm_bits_kernel, false, true)
LLMINT8_GEMM_KERNEL(llmint8_gemm_pair_bits_kernel, true, true)
#undef LLMINT8_GEMM_KERNEL

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
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

// 2-D row-major map over [rows, cols] elements with a (box_cols x box_rows) box, 128 B swizzle.
bool make_map(CUtensorMap *tm, const void *base, CUtensorMapDataType dt, int elem_bytes,
              int64_t cols, int64_t rows, int64_t pitch_elems, uint32_t box_cols,
              uint32_t box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(pitch_elems * elem_bytes)};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return enc(tm, dt, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct DeviceInfo {
    int sms = 0;
    bool attr_set = false;
};

// The CTA-pair kernel takes every call with more than 128 rows of X.
bool use_pair(int64_t M) { return M > BM; }

}  // namespace

cudaError_t launch_gemm(const GemmLaunch &g, cudaStream_t s) {
    static std::mutex mu;
    static DeviceInfo info[64];
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    int sms;
    {
        std::lock_guard<std::mutex> lk(mu);
        DeviceInfo &d = info[dev];
        if (!d.attr_set) {
            err = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
            if (err != cudaSuccess) return err;
            for (auto k : {llmint8_gemm_kernel, llmint8_gemm_bits_kernel}) {
                err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           smem_bytes<false>());
                if (err != cudaSuccess) return err;
            }
            for (auto k : {llmint8_gemm_pair_kernel, llmint8_gemm_pair_bits_kernel}) {
                err = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           smem_bytes<true>());
                if (err != cudaSuccess) return err;
            }
            d.attr_set = true;
        }
        sms = d.sms;
    }
    const bool pair = use_pair(g.M);
    const uint32_t b_rows = pair ? (uint32_t)Cfg<true>::B_ROWS : (uint32_t)Cfg<false>::B_ROWS;
    CUtensorMap tmA, tmB, tmXo, tmWo;
    memset(&tmXo, 0, sizeof(tmXo));
    memset(&tmWo, 0, sizeof(tmWo));
    bool ok = make_map(&tmA, g.Xq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.K, g.M, g.K, BKB, BM) &&
              make_map(&tmB, g.CB, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, g.K, g.N, g.K, BKB, b_rows);
    if (ok && g.cap > 0)
        ok = make_map(&tmXo, g.Xo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, g.pitch, g.M, g.pitch,
                      BKB / 2, BM) &&
             make_map(&tmWo, g.Wo, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, g.pitch, g.N, g.pitch,
                      BKB / 2, b_rows);
    if (!ok) return cudaErrorInvalidValue;
    Args a;
    a.Xo = g.Xo;
    a.Wo = g.Wo;
    a.pitch = (int)g.pitch;
    a.count = g.count;
    a.cap = g.cap;
    a.SCA = g.SCA;
    a.SCB = g.SCB;
    a.bias = g.bias;
    a.Y = g.Y;
    a.C_debug = g.C_debug;
    a.ybits = g.ybits;
    a.ybits_words = (int)ceil_div(g.N, 32);
    a.ytf = g.ybits && g.ythreshold > 0.0f ? fp16_rounded_threshold_f32(g.ythreshold) : 0.0f;
    a.ybits_all = g.ybits && g.ythreshold <= 0.0f ? 1 : 0;
    a.status = g.status;
    a.M = (int)g.M;
    a.N = (int)g.N;
    a.K = (int)g.K;
    a.num_kb = (int)ceil_div(g.K, BKB);
    a.tiles_m = (int)ceil_div(g.M, pair ? 2 * BM : BM);
    a.tiles_n = (int)ceil_div(g.N, BN);
    a.timeout_ns = g.timeout_ns;
    const int tiles = a.tiles_m * a.tiles_n;
    // one CTA (or one pair of CTAs) per tile, persistent beyond the SM count
    const int grid = pair ? 2 * std::min(tiles, sms / 2) : std::min(tiles, sms);
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 2;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = (size_t)(pair ? smem_bytes<true>() : smem_bytes<false>());
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pair ? 2 : 1;
    auto kernel = pair ? (g.ybits ? llmint8_gemm_pair_bits_kernel : llmint8_gemm_pair_kernel)
                       : (g.ybits ? llmint8_gemm_bits_kernel : llmint8_gemm_kernel);
    err = cudaLaunchKernelEx(&cfg, kernel, tmA, tmB, tmXo, tmWo, a);
    note_launches(1);
    return err != cudaSuccess ? err : cudaGetLastError();
}

}  // namespace llmint8

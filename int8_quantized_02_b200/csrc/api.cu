// C ABI of the LLM.int8() layer: argument checks, workspace layout and kernel launches.
// Declarations and the contract of every entry point are in include/llmint8.h.
#include <math.h>
#include <string.h>

#include <unistd.h>

#include <atomic>
#include <chrono>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

using namespace llmint8;

namespace {

// An NVTX range (domain "llmint8", named after the entry point) around every call that
// launches work, so that a profiler's timeline shows the layer's calls.  Without a tool
// attached it costs a pointer test.
class CallRange {
  public:
    explicit CallRange(const char *name) {
        nvtxEventAttributes_t e = {};
        e.version = NVTX_VERSION;
        e.size = NVTX_EVENT_ATTRIB_STRUCT_SIZE;
        e.messageType = NVTX_MESSAGE_TYPE_ASCII;
        e.message.ascii = name;
        nvtxDomainRangePushEx(domain(), &e);
    }
    ~CallRange() { nvtxDomainRangePop(domain()); }
    CallRange(const CallRange &) = delete;
    CallRange &operator=(const CallRange &) = delete;

  private:
    static nvtxDomainHandle_t domain() {
        static const nvtxDomainHandle_t d = nvtxDomainCreateA("llmint8");
        return d;
    }
};
#define LLMINT8_CALL_RANGE() CallRange llmint8_call_range_(__func__)

constexpr uint64_t kDefaultTimeoutNs = 1000000000ull;
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
std::atomic<uint64_t> g_launches{0};
// The first call number of this process: in [1, 2^31), mixed from the clock and the process
// id, so that call-tagged words another process left in the same device memory (workspaces are
// not cleared) are unlikely to carry a number this process uses.
unsigned long long first_epoch() {
    unsigned long long x =
        (unsigned long long)std::chrono::steady_clock::now().time_since_epoch().count();
    x ^= (unsigned long long)getpid() * 0x9e3779b97f4a7c15ull;
    x ^= x >> 29;
    x *= 0xbf58476d1ce4e5b9ull;
    x ^= x >> 32;
    return 1ull + (x & 0x7ffffffeull);
}
std::atomic<unsigned long long> g_epoch{first_epoch()};   // one per call that writes a status word

StatusRef next_status(WsHeader *h) {
    return StatusRef{&h->status, &h->timeout, g_epoch.fetch_add(1) << 4};
}
std::atomic<cudaEvent_t> g_prof_start{nullptr}, g_prof_stop{nullptr};

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bool shape_ok_mk(int64_t M, int64_t K) {
    return M >= 1 && M <= (int64_t)INT32_MAX && K >= 16 && K % 16 == 0 && K <= 131072;
}
bool shape_ok_n(int64_t N) { return N >= 16 && N % 16 == 0 && N <= (int64_t)INT32_MAX; }

// Workspace of llmint8_linear, every region 256-byte aligned.
struct LinearLayout {
    ScanPlan plan;
    int64_t cap = 0, pitch = 0;
    size_t partial = 0, bitmap = 0, idx = 0, sca = 0, xq = 0, xo = 0, wo = 0, total = 0;
    size_t dtable = 0, dimage = 0;    // decode path (shapes with M <= 16, K <= 16384 only)
};

LinearLayout linear_layout(int64_t M, int64_t N, int64_t K, int64_t cap) {
    LinearLayout L;
    L.plan = scan_plan(M, K);
    L.cap = cap;
    L.pitch = align_up(cap, 64);
    size_t off = sizeof(WsHeader);
    auto take = [&](size_t bytes) {
        size_t at = off;
        off = (size_t)align_up((int64_t)(off + bytes), 256);
        return at;
    };
    L.partial = take((size_t)(L.plan.splits * L.plan.nwords) * 4);
    L.bitmap = take((size_t)L.plan.nwords * 4);
    L.idx = take((size_t)std::max<int64_t>(cap, 1) * 4);
    L.sca = take((size_t)M * 4);
    L.xq = take((size_t)(M * K));
    L.xo = take((size_t)(M * L.pitch) * 2);
    L.wo = take((size_t)(N * L.pitch) * 2);
    if (M <= kDecodeMaxM && K <= kDecodeMaxK) {
        L.dtable = take(sizeof(DecodeTable));
        off = (size_t)align_up((int64_t)off, 1024);
        L.dimage = take((size_t)decode_image_bytes(M, K));
    }
    L.total = off;
    return L;
}

struct QuantLayout {
    ScanPlan plan;
    size_t partial = 0, bitmap = 0, idx = 0, total = 0;
};

// Workspace of llmint8_quantize_rows_and_find_outliers and llmint8_outlier_bitmap (the
// latter also lists every outlier column, so the capacity never runs out there).
QuantLayout quant_layout(int64_t M, int64_t K) {
    QuantLayout L;
    L.plan = scan_plan(M, K);
    size_t off = sizeof(WsHeader);
    L.partial = off;
    off = (size_t)align_up((int64_t)(off + (size_t)(L.plan.splits * L.plan.nwords) * 4), 256);
    L.bitmap = off;
    off = (size_t)align_up((int64_t)(off + (size_t)L.plan.nwords * 4), 256);
    L.idx = off;
    off = (size_t)align_up((int64_t)(off + (size_t)K * 4), 256);
    L.total = off;
    return L;
}

template <class T>
T *at(void *ws, size_t off) {
    return reinterpret_cast<T *>(static_cast<uint8_t *>(ws) + off);
}

// Profile events become real event-record nodes when the call is captured into a CUDA
// graph (a plain record inside stream capture only expresses a dependency).
cudaError_t record_profile_event(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(s, &cs);
    if (e != cudaSuccess) return e;
    return cs == cudaStreamCaptureStatusActive
               ? cudaEventRecordWithFlags(ev, s, cudaEventRecordExternal)
               : cudaEventRecord(ev, s);
}

llmint8_status from_cuda(cudaError_t e) { return e == cudaSuccess ? LLMINT8_OK : LLMINT8_ERR_CUDA; }

// The decode path covers few activation rows and an X whose quantized image fits in shared
// memory; threshold <= 0 (every column fp16) goes through the GEMM path.
bool use_decode_path(int64_t M, int64_t K, float threshold, int64_t cap) {
    return M <= kDecodeMaxM && K <= kDecodeMaxK && threshold > 0.0f &&
           cap <= kDecodeMaxOutliers;
}

// Arguments of a decode-path launch whose status words live in the header `h`.
DecodeLaunch decode_launch(const uint16_t *X, int64_t M, int64_t K, const int8_t *CB,
                           const float *SCB, int64_t N, const uint16_t *bias,
                           const uint16_t *W_fp16, float threshold, int64_t cap, uint16_t *Y,
                           int32_t *C_debug, WsHeader *h, DecodeTable *table,
                           uint8_t *image, StatusRef status) {
    DecodeLaunch d;
    d.X = reinterpret_cast<const __half *>(X);
    d.CB = CB;
    d.SCB = SCB;
    d.W16 = reinterpret_cast<const __half *>(W_fp16);
    d.bias = reinterpret_cast<const __half *>(bias);
    d.Y = reinterpret_cast<__half *>(Y);
    d.C_debug = C_debug;
    d.Wo = nullptr;
    d.wo_pitch = 0;
    d.bitmaps = nullptr;
    d.n_bitmaps = 0;
    d.ybits = nullptr;
    d.ythreshold = 0.0f;
    d.count = &h->n_outliers;
    d.table = table;
    d.image = image;
    d.status = status;
    d.M = M;
    d.N = N;
    d.K = K;
    d.cap = cap;
    d.threshold = threshold;
    d.timeout_ns = g_timeout_ns.load();
    return d;
}

// launch_decode between the process-wide profile events (when set).
llmint8_status run_decode(const DecodeLaunch &d, cudaStream_t s) {
    cudaEvent_t ev0 = g_prof_start.load(), ev1 = g_prof_stop.load();
    if (ev0 && record_profile_event(ev0, s) != cudaSuccess) return LLMINT8_ERR_CUDA;
    if (launch_decode(d, s) != cudaSuccess) return LLMINT8_ERR_CUDA;
    if (ev1 && record_profile_event(ev1, s) != cudaSuccess) return LLMINT8_ERR_CUDA;
    return LLMINT8_OK;
}

// launch_gemm between the process-wide profile events (when set).
llmint8_status run_gemm(const GemmLaunch &g, cudaStream_t s) {
    cudaEvent_t ev0 = g_prof_start.load(), ev1 = g_prof_stop.load();
    if (ev0 && record_profile_event(ev0, s) != cudaSuccess) return LLMINT8_ERR_CUDA;
    if (launch_gemm(g, s) != cudaSuccess) return LLMINT8_ERR_CUDA;
    if (ev1 && record_profile_event(ev1, s) != cudaSuccess) return LLMINT8_ERR_CUDA;
    return LLMINT8_OK;
}

}  // namespace

void llmint8::note_launches(int n) { g_launches.fetch_add((uint64_t)n); }

extern "C" {

llmint8_status llmint8_set_profile_events(void *start, void *stop) {
    if ((start == nullptr) != (stop == nullptr)) return LLMINT8_ERR_INVALID_ARG;
    g_prof_start.store(static_cast<cudaEvent_t>(start));
    g_prof_stop.store(static_cast<cudaEvent_t>(stop));
    return LLMINT8_OK;
}

uint64_t llmint8_kernel_launch_count(void) { return g_launches.load(); }


const char *llmint8_status_string(llmint8_status s) {
    switch (s) {
        case LLMINT8_OK: return "ok";
        case LLMINT8_ERR_INVALID_ARG: return "invalid argument";
        case LLMINT8_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case LLMINT8_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case LLMINT8_ERR_OUTLIER_CAPACITY: return "more outlier columns than the capacity";
        case LLMINT8_ERR_TIMEOUT: return "a bounded wait in a kernel timed out";
        case LLMINT8_ERR_CUDA: return "CUDA error";
        case LLMINT8_ERR_DEVICE_CHECK: return "a device-side bounds check failed (debug build)";
    }
    return "unknown status";
}

int llmint8_build_flags(void) {
#ifdef LLMINT8_DEBUG
    return 1;
#else
    return 0;
#endif
}

llmint8_status llmint8_set_wait_timeout_ns(uint64_t ns) {
    g_timeout_ns.store(ns == 0 ? kDefaultTimeoutNs : ns);
    return LLMINT8_OK;
}

size_t llmint8_quantize_workspace_size(int64_t M, int64_t K) {
    if (!shape_ok_mk(M, K)) return 0;
    return quant_layout(M, K).total;
}

size_t llmint8_linear_workspace_size(int64_t M, int64_t N, int64_t K, int64_t max_outliers) {
    if (!shape_ok_mk(M, K) || !shape_ok_n(N) || max_outliers < 0 || max_outliers > K) return 0;
    return linear_layout(M, N, K, max_outliers).total;
}

llmint8_status llmint8_quantize_weight_colwise(const uint16_t *W, int64_t N, int64_t K,
                                               int8_t *CB, float *SCB, void *stream) {
    LLMINT8_CALL_RANGE();
    if (!W || !CB || !SCB) return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(CB) || !aligned4(SCB)) return LLMINT8_ERR_INVALID_ARG;
    if (!shape_ok_mk(N, K)) return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    return from_cuda(launch_quantize_weight(reinterpret_cast<const __half *>(W), N, K, CB, SCB,
                                            static_cast<cudaStream_t>(stream)));
}

llmint8_status llmint8_dequant(const int8_t *CB, const float *SCB, int64_t N, int64_t K,
                               uint16_t *W_out, void *stream) {
    LLMINT8_CALL_RANGE();
    if (!CB || !SCB || !W_out) return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(CB) || !aligned16(W_out) || !aligned4(SCB)) return LLMINT8_ERR_INVALID_ARG;
    if (!shape_ok_mk(N, K)) return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    return from_cuda(launch_dequant(CB, SCB, N, K, reinterpret_cast<__half *>(W_out),
                                    static_cast<cudaStream_t>(stream)));
}

llmint8_status llmint8_quantize_rows_and_find_outliers(const uint16_t *X, int64_t M, int64_t K,
                                                       float threshold, int8_t *Xq, float *SCA,
                                                       int32_t *outlier_idx, int32_t *n_outliers,
                                                       int64_t cap, void *ws, size_t ws_bytes,
                                                       void *stream) {
    LLMINT8_CALL_RANGE();
    if (!X || !Xq || !SCA || !n_outliers || !ws || (cap > 0 && !outlier_idx))
        return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(Xq) || !aligned4(SCA) || !aligned4(n_outliers) ||
        !aligned16(ws) || (outlier_idx && !aligned4(outlier_idx)))
        return LLMINT8_ERR_INVALID_ARG;
    if (isnan(threshold)) return LLMINT8_ERR_INVALID_ARG;
    if (!shape_ok_mk(M, K)) return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (cap < 0 || cap > K) return LLMINT8_ERR_INVALID_ARG;
    const QuantLayout L = quant_layout(M, K);
    if (ws_bytes < L.total) return LLMINT8_ERR_WORKSPACE_TOO_SMALL;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsHeader *h = at<WsHeader>(ws, 0);
    const __half *Xh = reinterpret_cast<const __half *>(X);
    uint32_t *bitmap = at<uint32_t>(ws, L.bitmap);
    cudaError_t e = launch_outlier_detect(Xh, M, K, threshold, L.plan, at<uint32_t>(ws, L.partial),
                                          bitmap, outlier_idx, cap, n_outliers, next_status(h), s);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    return from_cuda(launch_quantize_rows(Xh, M, K, bitmap, outlier_idx, n_outliers, cap, 0, Xq,
                                          SCA, nullptr, nullptr, nullptr, nullptr, 0, nullptr, s));
}

}  // extern "C"

namespace {

// Every check of llmint8_linear that needs no CUDA call, in the order the header lists them.
llmint8_status check_linear(const uint16_t *X, int64_t M, int64_t K, const int8_t *CB,
                            const float *SCB, int64_t N, const uint16_t *bias,
                            const uint16_t *W_fp16, float threshold, int64_t max_outliers,
                            const uint16_t *Y, const void *ws, size_t ws_bytes,
                            const int32_t *C_debug) {
    if (!X || !CB || !SCB || !Y || !ws) return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(CB) || !aligned16(SCB) || !aligned16(Y) || !aligned16(ws) ||
        (bias && !aligned16(bias)) || (W_fp16 && !aligned16(W_fp16)) ||
        (C_debug && !aligned16(C_debug)))
        return LLMINT8_ERR_INVALID_ARG;
    if (isnan(threshold)) return LLMINT8_ERR_INVALID_ARG;
    if (!shape_ok_mk(M, K) || !shape_ok_n(N)) return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (max_outliers < 0 || max_outliers > K) return LLMINT8_ERR_INVALID_ARG;
    if (ws_bytes < linear_layout(M, N, K, max_outliers).total)
        return LLMINT8_ERR_WORKSPACE_TOO_SMALL;
    return LLMINT8_OK;
}

// Arguments of the GEMM launch of a layer call whose workspace `ws` has layout L.
GemmLaunch gemm_launch(const LinearLayout &L, void *ws, const int8_t *CB, const float *SCB,
                       const uint16_t *bias, uint16_t *Y, int32_t *C_debug, StatusRef status,
                       int64_t M, int64_t N, int64_t K, int64_t max_outliers) {
    GemmLaunch g;
    g.Xq = at<int8_t>(ws, L.xq);
    g.CB = CB;
    g.Xo = at<__half>(ws, L.xo);
    g.Wo = at<__half>(ws, L.wo);
    g.pitch = L.pitch;
    g.count = &at<WsHeader>(ws, 0)->n_outliers;
    g.cap = max_outliers;
    g.SCA = at<float>(ws, L.sca);
    g.SCB = SCB;
    g.bias = reinterpret_cast<const __half *>(bias);
    g.Y = reinterpret_cast<__half *>(Y);
    g.C_debug = C_debug;
    g.ybits = nullptr;
    g.ythreshold = 0.0f;
    g.status = status;
    g.M = M;
    g.N = N;
    g.K = K;
    g.timeout_ns = g_timeout_ns.load();
    return g;
}

// Upper bound of the bitmaps one llmint8_linear_with_bitmaps call merges (ranks).
constexpr int64_t kMaxBitmaps = 65536;

// llmint8_linear, and with ybits non-null also the outlier bitmaps of Y for the next layer
// (llmint8_linear_next_bitmaps).
llmint8_status linear_call(const uint16_t *X, int64_t M, int64_t K, const int8_t *CB,
                           const float *SCB, int64_t N, const uint16_t *bias,
                           const uint16_t *W_fp16, float threshold, int64_t max_outliers,
                           uint16_t *Y, void *ws, size_t ws_bytes, void *stream,
                           int32_t *C_debug, uint32_t *ybits, float ythreshold) {
    const llmint8_status chk = check_linear(X, M, K, CB, SCB, N, bias, W_fp16, threshold,
                                            max_outliers, Y, ws, ws_bytes, C_debug);
    if (chk != LLMINT8_OK) return chk;
    const LinearLayout L = linear_layout(M, N, K, max_outliers);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsHeader *h = at<WsHeader>(ws, 0);
    const StatusRef status = next_status(h);
    const __half *Xh = reinterpret_cast<const __half *>(X);
    cudaError_t e;

    if (use_decode_path(M, K, threshold, max_outliers)) {
        // one weight-streaming tcgen05 kernel; every CTA quantizes X itself
        DecodeLaunch d = decode_launch(X, M, K, CB, SCB, N, bias, W_fp16, threshold,
                                       max_outliers, Y, C_debug, h,
                                       at<DecodeTable>(ws, L.dtable), at<uint8_t>(ws, L.dimage),
                                       status);
        if (C_debug) {
            d.Wo = at<__half>(ws, L.wo);
            d.wo_pitch = L.pitch;
        }
        d.ybits = ybits;
        d.ythreshold = ythreshold;
        return run_decode(d, s);
    }

    uint32_t *bitmap = at<uint32_t>(ws, L.bitmap);
    int32_t *idx = at<int32_t>(ws, L.idx);
    float *SCA = at<float>(ws, L.sca);
    int8_t *Xq = at<int8_t>(ws, L.xq);
    __half *Xo = at<__half>(ws, L.xo);
    __half *Wo = at<__half>(ws, L.wo);

    e = launch_outlier_detect(Xh, M, K, threshold, L.plan, at<uint32_t>(ws, L.partial),
                              bitmap,
                              idx, max_outliers, &h->n_outliers, status, s);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    e = launch_quantize_rows(Xh, M, K, bitmap, idx, &h->n_outliers, max_outliers, L.pitch, Xq, SCA,
                             max_outliers > 0 ? Xo : nullptr, CB, SCB,
                             reinterpret_cast<const __half *>(W_fp16), N,
                             max_outliers > 0 ? Wo : nullptr, s);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    GemmLaunch g = gemm_launch(L, ws, CB, SCB, bias, Y, C_debug, status, M, N, K, max_outliers);
    g.ybits = ybits;
    g.ythreshold = ythreshold;
    return run_gemm(g, s);
}

}  // namespace

extern "C" {

llmint8_status llmint8_linear(const uint16_t *X, int64_t M, int64_t K, const int8_t *CB,
                              const float *SCB, int64_t N, const uint16_t *bias,
                              const uint16_t *W_fp16, float threshold, int64_t max_outliers,
                              uint16_t *Y, void *ws, size_t ws_bytes, void *stream,
                              int32_t *C_debug) {
    LLMINT8_CALL_RANGE();
    return linear_call(X, M, K, CB, SCB, N, bias, W_fp16, threshold, max_outliers, Y, ws,
                       ws_bytes, stream, C_debug, nullptr, 0.0f);
}

llmint8_status llmint8_linear_next_bitmaps(const uint16_t *X, int64_t M, int64_t K,
                                           const int8_t *CB, const float *SCB, int64_t N,
                                           const uint16_t *bias, const uint16_t *W_fp16,
                                           float threshold, int64_t max_outliers, uint16_t *Y,
                                           void *ws, size_t ws_bytes, void *stream,
                                           int32_t *C_debug, float next_threshold,
                                           uint32_t *next_bitmaps) {
    LLMINT8_CALL_RANGE();
    if (!next_bitmaps || !aligned4(next_bitmaps) || isnan(next_threshold))
        return LLMINT8_ERR_INVALID_ARG;
    return linear_call(X, M, K, CB, SCB, N, bias, W_fp16, threshold, max_outliers, Y, ws,
                       ws_bytes, stream, C_debug, next_bitmaps, next_threshold);
}

llmint8_status llmint8_outlier_bitmap(const uint16_t *X, int64_t M, int64_t K, float threshold,
                                     uint32_t *bitmap, void *ws, size_t ws_bytes, void *stream) {
    LLMINT8_CALL_RANGE();
    if (!X || !bitmap || !ws) return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned4(bitmap) || !aligned16(ws)) return LLMINT8_ERR_INVALID_ARG;
    if (isnan(threshold)) return LLMINT8_ERR_INVALID_ARG;
    if (!shape_ok_mk(M, K)) return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    const QuantLayout L = quant_layout(M, K);
    if (ws_bytes < L.total) return LLMINT8_ERR_WORKSPACE_TOO_SMALL;
    WsHeader *h = at<WsHeader>(ws, 0);
    return from_cuda(launch_outlier_detect(reinterpret_cast<const __half *>(X), M, K, threshold,
                                           L.plan, at<uint32_t>(ws, L.partial),
                                           bitmap,
                                           at<int32_t>(ws, L.idx), K, &h->n_outliers,
                                           next_status(h), static_cast<cudaStream_t>(stream)));
}

llmint8_status llmint8_linear_with_bitmaps(const uint16_t *X, int64_t M, int64_t K,
                                           const int8_t *CB, const float *SCB, int64_t N,
                                           const uint16_t *bias, const uint16_t *W_fp16,
                                           const uint32_t *bitmaps, int64_t n_bitmaps,
                                           int64_t max_outliers, uint16_t *Y, void *ws,
                                           size_t ws_bytes, void *stream, int32_t *C_debug) {
    LLMINT8_CALL_RANGE();
    if (!bitmaps || !aligned4(bitmaps)) return LLMINT8_ERR_INVALID_ARG;
    if (n_bitmaps < 1 || n_bitmaps > kMaxBitmaps) return LLMINT8_ERR_INVALID_ARG;
    // the threshold plays no part: 6 only satisfies the shared checks
    const llmint8_status chk = check_linear(X, M, K, CB, SCB, N, bias, W_fp16, 6.0f,
                                            max_outliers, Y, ws, ws_bytes, C_debug);
    if (chk != LLMINT8_OK) return chk;
    const LinearLayout L = linear_layout(M, N, K, max_outliers);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    WsHeader *h = at<WsHeader>(ws, 0);
    const __half *Xh = reinterpret_cast<const __half *>(X);
    const StatusRef status = next_status(h);
    if (use_decode_path(M, K, 6.0f, max_outliers)) {
        // few rows: the decode kernel, its outlier columns taken from the merged bitmaps
        DecodeLaunch d = decode_launch(X, M, K, CB, SCB, N, bias, W_fp16, 6.0f, max_outliers,
                                       Y, C_debug, h, at<DecodeTable>(ws, L.dtable),
                                       at<uint8_t>(ws, L.dimage), status);
        d.bitmaps = bitmaps;
        d.n_bitmaps = n_bitmaps;
        if (C_debug) {
            d.Wo = at<__half>(ws, L.wo);
            d.wo_pitch = L.pitch;
        }
        return run_decode(d, s);
    }
    uint32_t *bitmap = at<uint32_t>(ws, L.bitmap);
    int32_t *idx = at<int32_t>(ws, L.idx);
    __half *Xo = at<__half>(ws, L.xo);
    __half *Wo = at<__half>(ws, L.wo);
    cudaError_t e = launch_outlier_merge(bitmaps, n_bitmaps, K, bitmap, idx, max_outliers,
                                         &h->n_outliers, status, s);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    e = launch_quantize_rows(Xh, M, K, bitmap, idx, &h->n_outliers, max_outliers, L.pitch,
                             at<int8_t>(ws, L.xq), at<float>(ws, L.sca),
                             max_outliers > 0 ? Xo : nullptr, CB, SCB,
                             reinterpret_cast<const __half *>(W_fp16), N,
                             max_outliers > 0 ? Wo : nullptr, s);
    if (e != cudaSuccess) return LLMINT8_ERR_CUDA;
    return run_gemm(gemm_launch(L, ws, CB, SCB, bias, Y, C_debug, status, M, N, K, max_outliers),
                    s);
}

llmint8_status llmint8_linear_host(const uint16_t *X_host, int64_t M, int64_t K,
                                   const int8_t *CB, const float *SCB, int64_t N,
                                   const uint16_t *bias, const uint16_t *W_fp16, float threshold,
                                   int64_t max_outliers, uint16_t *Y_host, uint16_t *X_dev,
                                   uint16_t *Y_dev, void *ws, size_t ws_bytes, void *stream) {
    LLMINT8_CALL_RANGE();
    if (!X_host || !Y_host) return LLMINT8_ERR_INVALID_ARG;
    const llmint8_status chk = check_linear(X_dev, M, K, CB, SCB, N, bias, W_fp16, threshold,
                                            max_outliers, Y_dev, ws, ws_bytes, nullptr);
    if (chk != LLMINT8_OK) return chk;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaMemcpyAsync(X_dev, X_host, (size_t)(M * K) * 2, cudaMemcpyHostToDevice, s) !=
        cudaSuccess)
        return LLMINT8_ERR_CUDA;
    const llmint8_status st = llmint8_linear(X_dev, M, K, CB, SCB, N, bias, W_fp16, threshold,
                                             max_outliers, Y_dev, ws, ws_bytes, stream, nullptr);
    if (st != LLMINT8_OK) return st;
    return from_cuda(
        cudaMemcpyAsync(Y_host, Y_dev, (size_t)(M * N) * 2, cudaMemcpyDeviceToHost, s));
}

llmint8_status llmint8_device_status(const void *ws, void *stream) {
    if (!ws) return LLMINT8_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    unsigned long long words[2] = {0, 0};   // status, timeout
    if (cudaMemcpy(words, ws, sizeof(words), cudaMemcpyDeviceToHost) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    // epochs are never 0: a zero-filled header has recorded no call and no timeout
    if ((words[0] >> 4) != 0 && (words[1] >> 4) == (words[0] >> 4))
        return static_cast<llmint8_status>(words[1] & 0xFull);
    return static_cast<llmint8_status>(words[0] & 0xFull);
}

llmint8_status llmint8_workspace_outlier_count(const void *ws, void *stream, int32_t *count) {
    if (!ws || !count) return LLMINT8_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    const WsHeader *h = static_cast<const WsHeader *>(ws);
    if (cudaMemcpy(count, &h->n_outliers, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return LLMINT8_ERR_CUDA;
    return LLMINT8_OK;
}

llmint8_status llmint8_workspace_outlier_weights(const void *ws, int64_t M, int64_t N, int64_t K,
                                                 int64_t max_outliers, uint16_t *Wo,
                                                 int64_t n_cols, void *stream) {
    LLMINT8_CALL_RANGE();
    if (!ws || !Wo || !aligned16(ws) || !aligned16(Wo)) return LLMINT8_ERR_INVALID_ARG;
    if (!shape_ok_mk(M, K) || !shape_ok_n(N)) return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (max_outliers < 0 || max_outliers > K || n_cols < 0 || n_cols > max_outliers)
        return LLMINT8_ERR_INVALID_ARG;
    if (n_cols == 0) return LLMINT8_OK;
    const LinearLayout L = linear_layout(M, N, K, max_outliers);
    return from_cuda(cudaMemcpy2DAsync(Wo, (size_t)n_cols * 2,
                                       static_cast<const uint8_t *>(ws) + L.wo,
                                       (size_t)L.pitch * 2, (size_t)n_cols * 2, (size_t)N,
                                       cudaMemcpyDeviceToDevice,
                                       static_cast<cudaStream_t>(stream)));
}

}  // extern "C"

// ------------------------------------------------------------------ no-allocation call ----
//
// llmint8_linear_noalloc runs the decode kernel with its scratch - the 256-byte header that
// receives the call's status words and outlier count, and the table of outlier columns and row
// scales and the int8 image of X that the kernel's first CTA hands to the others - in this
// file-scope device array (about 260 KiB) instead of a caller workspace.  It is meant for callers that cannot allocate device memory
// at the call site: a token-by-token decode loop that must not call cudaMalloc or cudaFree
// between steps (cudaFree waits for the whole device), and plain C hosts that hold no device
// allocator of their own.  Nothing here allocates: no cudaMalloc, cudaFree or allocating
// library routine.
//
// Nothing in it needs clearing between calls: every call tags its status words and its table
// with a fresh call epoch (the counter only grows and starts above zero), and the outlier
// count is plain-stored by each call.  Calls in stream order are safe: the decode kernel of a
// call writes the scratch only after the previous grid on its stream has finished.  Calls
// that overlap - on two streams, or from two host threads without stream order between them -
// share the one scratch of their device and race on its table; their outputs are undefined.
namespace {

// the header, the table (256-byte aligned), then the operand image (1024-byte aligned) of the
// largest decode shape: 16 rows x 16384 columns
constexpr size_t kNoAllocTableOffset = sizeof(WsHeader);
constexpr size_t kNoAllocImageOffset =
    (size_t)align_up((int64_t)(kNoAllocTableOffset + sizeof(DecodeTable)), 1024);
constexpr size_t kNoAllocScratchBytes =
    kNoAllocImageOffset + (size_t)decode_image_bytes(kDecodeMaxM, kDecodeMaxK);

__device__ __align__(1024) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kNoAllocMaxDevices = 64;
std::mutex g_noalloc_mu;
void *g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Set-up, once per device, with that device current: the scratch's device address (the
// array's name in host code is only a host-side stand-in).  The address is cached for the
// life of the process; a device reset (cudaDeviceReset) invalidates it and is not supported
// between calls of this entry point.
cudaError_t noalloc_scratch(void **ptr) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (g_noalloc_ptr[dev] == nullptr) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_noalloc_ptr[dev] = p;
    }
    *ptr = g_noalloc_ptr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" {

llmint8_status llmint8_linear_noalloc(const uint16_t *X, int64_t M, int64_t K, const int8_t *CB,
                                      const float *SCB, int64_t N, const uint16_t *bias,
                                      const uint16_t *W_fp16, float threshold,
                                      int64_t max_outliers, uint16_t *Y, void *stream,
                                      void **scratch_out) {
    LLMINT8_CALL_RANGE();
    if (!X || !CB || !SCB || !Y) return LLMINT8_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(CB) || !aligned16(SCB) || !aligned16(Y) ||
        (bias && !aligned16(bias)) || (W_fp16 && !aligned16(W_fp16)))
        return LLMINT8_ERR_INVALID_ARG;
    if (isnan(threshold)) return LLMINT8_ERR_INVALID_ARG;
    if (!shape_ok_mk(M, K) || !shape_ok_n(N)) return LLMINT8_ERR_UNSUPPORTED_SHAPE;
    if (max_outliers < 0 || max_outliers > K) return LLMINT8_ERR_INVALID_ARG;
    // only what the decode path covers runs without a workspace
    if (!use_decode_path(M, K, threshold, max_outliers)) return LLMINT8_ERR_UNSUPPORTED_SHAPE;

    void *base = nullptr;
    if (noalloc_scratch(&base) != cudaSuccess) return LLMINT8_ERR_CUDA;
    WsHeader *h = at<WsHeader>(base, 0);
    const DecodeLaunch d = decode_launch(X, M, K, CB, SCB, N, bias, W_fp16, threshold,
                                         max_outliers, Y, nullptr, h,
                                         at<DecodeTable>(base, kNoAllocTableOffset),
                                         at<uint8_t>(base, kNoAllocImageOffset), next_status(h));
    if (scratch_out) *scratch_out = base;
    return run_decode(d, static_cast<cudaStream_t>(stream));
}

}  // extern "C"

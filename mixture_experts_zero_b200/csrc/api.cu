// api.cu -- the extern "C" entry points of libmoezero.so (declared in include/lc_moe.h).
//
// Host side only: argument and shape checks (before any CUDA call), workspace carving, and the
// launch sequence of the layer on the caller's stream. The library allocates nothing; the only
// synchronising call is lc_moe_read_status.
#include <atomic>
#include <mutex>

#include "common.cuh"

namespace lcmoe {

namespace {

std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};
std::atomic<unsigned long long*> g_clock_probe{nullptr};

constexpr size_t kAlign = 256;
constexpr size_t kStatusBytes = 256;

size_t align_up(size_t v) { return (v + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_shape(const lc_moe_shape* s) {
    if (!s) return LC_MOE_ERR_INVALID_ARG;
    const int64_t E = static_cast<int64_t>(s->N) + s->Z;
    if (s->T < 0 || s->d < 64 || s->d % 64 || s->I < 64 || s->I % 64 || s->N < 1 || s->Z < 0 ||
        s->K < 1 || s->K > 32 || E < s->K || E > 2048)
        return LC_MOE_ERR_UNSUPPORTED_SHAPE;
    if (static_cast<int64_t>(s->T) * s->K >= (int64_t(1) << 31)) return LC_MOE_ERR_UNSUPPORTED_SHAPE;
    // row coordinates of the expert-weight tensor maps are 32-bit
    if (static_cast<int64_t>(s->N) * 2 * s->I >= (int64_t(1) << 31) ||
        static_cast<int64_t>(s->N) * s->d >= (int64_t(1) << 31))
        return LC_MOE_ERR_UNSUPPORTED_SHAPE;
    return LC_MOE_OK;
}

// Byte offsets of the forward workspace regions.
struct FwdLayout {
    size_t logits, idx, gate, offsets, row_token, pair_row, scratch, xq, sx, s_row, x_perm, h, hq, s_h, y,
        total;
    int64_t rows_cap;
};

// f8: the E4M3 variant (quantised token rows [T, d] bytes and their scales [T], grouped rows of
// d bytes with their scales [rows_cap], quantised H rows [rows_cap, I] bytes with their scales);
// otherwise grouped rows of d bf16 values.
FwdLayout fwd_layout(const lc_moe_shape* s, bool f8 = false) {
    FwdLayout L{};
    const size_t T = s->T, K = s->K, E = static_cast<size_t>(s->N) + s->Z;
    const int64_t rows_cap = static_cast<int64_t>(s->T) * (s->K < s->N ? s->K : s->N);
    size_t o = kStatusBytes;
    L.logits = o;    o = align_up(o + T * E * 4);
    L.idx = o;       o = align_up(o + T * K * 4);
    L.gate = o;      o = align_up(o + T * K * 4);
    L.offsets = o;   o = align_up(o + (static_cast<size_t>(s->N) + 1) * 4);
    L.row_token = o; o = align_up(o + T * K * 4);
    L.pair_row = o;  o = align_up(o + T * K * 4);
    L.scratch = o;   o = align_up(o + permute_scratch_bytes(s->T, s->N));
    if (f8) {
        L.xq = o;    o = align_up(o + T * s->d);
        L.sx = o;    o = align_up(o + T * 4);
        L.s_row = o; o = align_up(o + static_cast<size_t>(rows_cap) * 4);
    }
    L.x_perm = o;    o = align_up(o + static_cast<size_t>(rows_cap) * s->d * (f8 ? 1 : 2));
    L.h = o;         o = align_up(o + static_cast<size_t>(rows_cap) * s->I * 2);
    if (f8) {
        L.hq = o;    o = align_up(o + static_cast<size_t>(rows_cap) * s->I);
        L.s_h = o;   o = align_up(o + static_cast<size_t>(rows_cap) * 4);
    }
    L.y = o;         o = align_up(o + static_cast<size_t>(rows_cap) * s->d * 2);
    L.total = o;
    L.rows_cap = rows_cap;
    return L;
}

size_t route_ws_bytes(const lc_moe_shape* s) {
    return kStatusBytes + align_up(static_cast<size_t>(s->T) * (static_cast<size_t>(s->N) + s->Z) * 4);
}

size_t permute_ws_bytes(const lc_moe_shape* s) {
    return kStatusBytes + align_up(permute_scratch_bytes(s->T, s->N));
}

template <class P>
P* at(void* ws, size_t off) {
    return reinterpret_cast<P*>(static_cast<char*>(ws) + off);
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? LC_MOE_OK : LC_MOE_ERR_CUDA; }

int device_ok() {
    const DevInfo* di = current_device_info();
    if (!di) return LC_MOE_ERR_CUDA;
    if (!di->ok_sm100) return LC_MOE_ERR_NOT_SM100;
    return LC_MOE_OK;
}

#define LC_TRY(expr)                            \
    do {                                        \
        const int lc_rc_ = (expr);              \
        if (lc_rc_ != LC_MOE_OK) return lc_rc_; \
    } while (0)

#define LC_CUDA(expr) LC_TRY(cuda_status(expr))

int record(void* const* events, int i, cudaStream_t st) {
    if (!events) return LC_MOE_OK;
    return cuda_status(cudaEventRecord(static_cast<cudaEvent_t>(events[i]), st));
}

int forward_impl(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                 const void* w13, const float* w13_scale, const void* w2, const float* w2_scale,
                 void* out, int32_t* idx, float* gate, int32_t* counts, void* ws, size_t ws_bytes,
                 void* stream, void* const* events) {
    // w13_scale != NULL selects the E4M3 experts (w13 and w2 then hold E4M3 codes)
    const bool f8 = w13_scale != nullptr;
    LC_TRY(check_shape(s));
    if (f8 && (s->d % 128 || s->I % 128)) return LC_MOE_ERR_UNSUPPORTED_SHAPE;
    if (!x || !wr || !bias || !w13 || !w2 || !out || !ws || (f8 && !w2_scale)) return LC_MOE_ERR_INVALID_ARG;
    const FwdLayout L = fwd_layout(s, f8);
    if (ws_bytes < L.total) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    for (const void* p : {x, wr, static_cast<const void*>(bias), w13, static_cast<const void*>(w13_scale), w2,
                          static_cast<const void*>(w2_scale), static_cast<const void*>(out),
                          static_cast<const void*>(idx), static_cast<const void*>(gate),
                          static_cast<const void*>(counts), static_cast<const void*>(ws)})
        if (p && !aligned16(p)) return LC_MOE_ERR_MISALIGNED;
    if (s->T == 0) return LC_MOE_OK;
    LC_TRY(device_ok());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int E = s->N + s->Z;
    uint32_t* status = at<uint32_t>(ws, 0);
    float* logits = at<float>(ws, L.logits);
    int32_t* idx_w = idx ? idx : at<int32_t>(ws, L.idx);
    float* gate_w = gate ? gate : at<float>(ws, L.gate);
    int32_t* offsets = at<int32_t>(ws, L.offsets);
    int32_t* row_token = at<int32_t>(ws, L.row_token);
    int32_t* pair_row = at<int32_t>(ws, L.pair_row);
    int32_t* scratch = at<int32_t>(ws, L.scratch);
    void* x_perm = at<void>(ws, L.x_perm);
    void* h = at<void>(ws, L.h);
    void* y = at<void>(ws, L.y);

    LC_TRY(record(events, LC_MOE_STAGE_ROUTER_GEMM, st));
    LC_CUDA(launch_router_gemm(x, wr, logits, s->T, s->d, E, status, st));
    LC_TRY(record(events, LC_MOE_STAGE_TOPK, st));
    LC_CUDA(launch_topk(logits, bias, s->T, E, s->K, idx_w, gate_w, counts, status, st));
    LC_TRY(record(events, LC_MOE_STAGE_PERMUTE, st));
    LC_CUDA(launch_permute(idx_w, s->T, s->K, s->N, E, offsets, row_token, pair_row, scratch, status, st));
    LC_TRY(record(events, LC_MOE_STAGE_GATHER, st));
    if (f8) {
        // quantise each token row once, then copy codes and scale to each of its FFN rows
        void* xq = at<void>(ws, L.xq);
        float* sx = at<float>(ws, L.sx);
        float* s_row = at<float>(ws, L.s_row);
        LC_CUDA(launch_quantize_rows_e4m3(x, s->T, s->d, xq, sx, st));
        LC_CUDA(launch_gather_e4m3(xq, sx, s->T, s->d, s->K, pair_row, x_perm, s_row, status, st));
        LC_TRY(record(events, LC_MOE_STAGE_GEMM1, st));
        LC_CUDA(launch_grouped_swiglu_e4m3(x_perm, s_row, L.rows_cap, offsets, s->N, w13, w13_scale, s->d,
                                           s->I, h, status, st));
    } else {
        LC_CUDA(launch_gather(x, s->T, s->d, s->K, pair_row, x_perm, status, st));
        LC_TRY(record(events, LC_MOE_STAGE_GEMM1, st));
        LC_CUDA(launch_grouped_swiglu(x_perm, L.rows_cap, offsets, s->N, w13, s->d, s->I, h, status, st));
    }
    LC_TRY(record(events, LC_MOE_STAGE_GEMM2, st));
    if (f8) {
        // quantise the offsets[N] rows of H that GEMM 1 wrote, one scale per row
        void* hq = at<void>(ws, L.hq);
        float* s_h = at<float>(ws, L.s_h);
        LC_CUDA(launch_quantize_rows_e4m3(h, L.rows_cap, s->I, hq, s_h, st, offsets + s->N));
        LC_CUDA(launch_grouped_down_e4m3(hq, s_h, L.rows_cap, offsets, s->N, w2, w2_scale, s->d, s->I, y,
                                         status, st));
    } else {
        LC_CUDA(launch_grouped_down(h, L.rows_cap, offsets, s->N, w2, s->d, s->I, y, status, st));
    }
    LC_TRY(record(events, LC_MOE_STAGE_COMBINE, st));
    LC_CUDA(launch_combine(x, y, gate_w, pair_row, s->T, s->d, s->K, out, st));
    LC_TRY(record(events, LC_MOE_NUM_STAGES, st));
    return LC_MOE_OK;
}

}  // namespace

const DevInfo* current_device_info() {
    static PerDeviceOnce query;
    static DevInfo infos[PerDeviceOnce::kMaxDevices];
    const cudaError_t e = query.run([](int dev) {
        int major = 0, minor = 0, sms = 0;
        cudaError_t r = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
        if (r == cudaSuccess) r = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
        if (r == cudaSuccess) r = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (r == cudaSuccess) {
            infos[dev].sm_count = sms;
            infos[dev].ok_sm100 = (major == 10 && minor == 0);
        }
        return r;
    });
    int dev = 0;
    if (e != cudaSuccess || cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return nullptr;
    }
    return &infos[dev];
}

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

unsigned long long* clock_probe() { return g_clock_probe.load(std::memory_order_relaxed); }

}  // namespace lcmoe

using namespace lcmoe;

extern "C" {

int32_t lc_moe_abi_version(void) { return LC_MOE_ABI_VERSION; }

const char* lc_moe_strerror(int code) {
    switch (code) {
        case LC_MOE_OK: return "ok";
        case LC_MOE_ERR_INVALID_ARG: return "invalid argument";
        case LC_MOE_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case LC_MOE_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case LC_MOE_ERR_NOT_SM100: return "device is not sm_100 (B200)";
        case LC_MOE_ERR_CUDA: return "CUDA error";
        case LC_MOE_ERR_DEVICE_STATUS: return "device status bits set";
        case LC_MOE_ERR_TIMEOUT: return "a bounded device wait timed out";
        case LC_MOE_ERR_MISALIGNED: return "pointer not 16-byte aligned";
        default: return "unknown error code";
    }
}

size_t lc_moe_workspace_bytes(const lc_moe_shape* s, int op) {
    if (check_shape(s) != LC_MOE_OK) return 0;
    switch (op) {
        case LC_MOE_OP_FORWARD: return fwd_layout(s).total;
        case LC_MOE_OP_FORWARD_FP8: return (s->d % 128 || s->I % 128) ? 0 : fwd_layout(s, true).total;
        case LC_MOE_OP_ROUTE: return route_ws_bytes(s);
        case LC_MOE_OP_PERMUTE: return permute_ws_bytes(s);
        case LC_MOE_OP_STATUS: return kStatusBytes;
        default: return 0;
    }
}

void lc_moe_set_wait_limit_ns(uint64_t limit_ns) {
    if (limit_ns < 1000000ull) limit_ns = 1000000ull;
    g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
}

void lc_moe_set_clock_probe(void* probe) {
    g_clock_probe.store(static_cast<unsigned long long*>(probe), std::memory_order_relaxed);
}

int lc_moe_check_wait_timeout(void* ws, size_t ws_bytes, void* stream) {
    if (!ws) return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws)) return LC_MOE_ERR_MISALIGNED;
    LC_TRY(device_ok());
    LC_CUDA(launch_wait_check(at<uint32_t>(ws, 0), wait_limit_ns(), static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_forward(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                   const void* w13, const void* w2, void* out, int32_t* idx, float* gate,
                   int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
    return forward_impl(s, x, wr, bias, w13, nullptr, w2, nullptr, out, idx, gate, counts, ws, ws_bytes, stream,
                        nullptr);
}

int lc_moe_forward_timed(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                         const void* w13, const void* w2, void* out, int32_t* idx, float* gate,
                         int32_t* counts, void* ws, size_t ws_bytes, void* stream,
                         void* const* events) {
    if (!events) return LC_MOE_ERR_INVALID_ARG;
    for (int i = 0; i <= LC_MOE_NUM_STAGES; ++i)
        if (!events[i]) return LC_MOE_ERR_INVALID_ARG;
    return forward_impl(s, x, wr, bias, w13, nullptr, w2, nullptr, out, idx, gate, counts, ws, ws_bytes, stream,
                        events);
}

int lc_moe_forward_fp8(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                       const void* w13q, const float* w13_scale, const void* w2q,
                       const float* w2_scale, void* out, int32_t* idx, float* gate, int32_t* counts,
                       void* ws, size_t ws_bytes, void* stream) {
    if (!w13_scale || !w2_scale) return LC_MOE_ERR_INVALID_ARG;
    return forward_impl(s, x, wr, bias, w13q, w13_scale, w2q, w2_scale, out, idx, gate, counts, ws,
                        ws_bytes, stream, nullptr);
}

int lc_moe_forward_fp8_timed(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                             const void* w13q, const float* w13_scale, const void* w2q,
                             const float* w2_scale, void* out, int32_t* idx, float* gate,
                             int32_t* counts, void* ws, size_t ws_bytes, void* stream,
                             void* const* events) {
    if (!w13_scale || !w2_scale || !events) return LC_MOE_ERR_INVALID_ARG;
    for (int i = 0; i <= LC_MOE_NUM_STAGES; ++i)
        if (!events[i]) return LC_MOE_ERR_INVALID_ARG;
    return forward_impl(s, x, wr, bias, w13q, w13_scale, w2q, w2_scale, out, idx, gate, counts, ws,
                        ws_bytes, stream, events);
}

int lc_moe_quantize_e4m3(const void* src, int64_t rows, int32_t cols, void* dst, float* scale,
                         void* stream) {
    if (rows < 0 || cols < 8 || cols % 8) return LC_MOE_ERR_INVALID_ARG;
    if (rows == 0) return LC_MOE_OK;
    if (!src || !dst || !scale) return LC_MOE_ERR_INVALID_ARG;
    if (!aligned16(src) || !aligned16(dst) || (reinterpret_cast<uintptr_t>(scale) & 3u))
        return LC_MOE_ERR_MISALIGNED;
    LC_TRY(device_ok());
    LC_CUDA(launch_quantize_rows_e4m3(src, rows, cols, dst, scale, static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_route(const lc_moe_shape* s, const void* x, const void* wr, const float* bias,
                 int32_t* idx, float* gate, int32_t* counts, float* logits, void* ws,
                 size_t ws_bytes, void* stream) {
    LC_TRY(check_shape(s));
    if (!x || !wr || !bias || !idx || !gate || !ws) return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < route_ws_bytes(s)) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    for (const void* p : {x, wr, static_cast<const void*>(bias), static_cast<const void*>(idx),
                          static_cast<const void*>(gate), static_cast<const void*>(counts),
                          static_cast<const void*>(logits), static_cast<const void*>(ws)})
        if (p && !aligned16(p)) return LC_MOE_ERR_MISALIGNED;
    if (s->T == 0) return LC_MOE_OK;
    LC_TRY(device_ok());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int E = s->N + s->Z;
    uint32_t* status = at<uint32_t>(ws, 0);
    float* z = logits ? logits : at<float>(ws, kStatusBytes);
    LC_CUDA(launch_router_gemm(x, wr, z, s->T, s->d, E, status, st));
    LC_CUDA(launch_topk(z, bias, s->T, E, s->K, idx, gate, counts, status, st));
    return LC_MOE_OK;
}

int lc_moe_bias_update(float* bias, int32_t* counts, int64_t T_all, int32_t N, int32_t Z,
                       int32_t K, int32_t K_e, float mu, int32_t reset_counts, void* stream) {
    if (!bias || !counts) return LC_MOE_ERR_INVALID_ARG;
    if (N < 1 || Z < 0 || K < 1 || K_e < 1 || K_e > K || T_all <= 0 || N + Z > (1 << 24) ||
        !(mu == mu))
        return LC_MOE_ERR_INVALID_ARG;
    if (!aligned16(bias) || !aligned16(counts)) return LC_MOE_ERR_MISALIGNED;
    LC_TRY(device_ok());
    LC_CUDA(launch_bias_update(bias, counts, N + Z, T_all, N, K, K_e, mu, reset_counts != 0,
                               static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_read_status(void* ws, uint32_t* status_out, void* stream) {
    if (!ws) return LC_MOE_ERR_INVALID_ARG;
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    uint32_t v = 0;
    LC_CUDA(cudaMemcpyAsync(&v, ws, sizeof v, cudaMemcpyDeviceToHost, st));
    LC_CUDA(cudaStreamSynchronize(st));
    if (v) {
        LC_CUDA(cudaMemsetAsync(ws, 0, sizeof v, st));
        LC_CUDA(cudaStreamSynchronize(st));
    }
    if (status_out) *status_out = v;
    if (v & LC_MOE_DEV_WAIT_TIMEOUT) return LC_MOE_ERR_TIMEOUT;
    return v ? LC_MOE_ERR_DEVICE_STATUS : LC_MOE_OK;
}

int lc_moe_router_logits(const lc_moe_shape* s, const void* x, const void* wr, float* logits,
                         void* ws, size_t ws_bytes, void* stream) {
    LC_TRY(check_shape(s));
    if (!x || !wr || !logits || !ws) return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    for (const void* p : {x, wr, static_cast<const void*>(logits), static_cast<const void*>(ws)})
        if (!aligned16(p)) return LC_MOE_ERR_MISALIGNED;
    if (s->T == 0) return LC_MOE_OK;
    LC_TRY(device_ok());
    LC_CUDA(launch_router_gemm(x, wr, logits, s->T, s->d, s->N + s->Z, at<uint32_t>(ws, 0),
                               static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_topk(const lc_moe_shape* s, const float* logits, const float* bias, int32_t* idx,
                float* gate, int32_t* counts, void* ws, size_t ws_bytes, void* stream) {
    LC_TRY(check_shape(s));
    if (!logits || !bias || !idx || !gate || !ws) return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    if (s->T == 0) return LC_MOE_OK;
    LC_TRY(device_ok());
    LC_CUDA(launch_topk(logits, bias, s->T, s->N + s->Z, s->K, idx, gate, counts,
                        at<uint32_t>(ws, 0), static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_expert_hist(const int32_t* idx, int64_t n, int32_t n_bins, int32_t* counts, void* ws,
                       size_t ws_bytes, void* stream) {
    if (!counts || !ws || n < 0 || n_bins < 1 || n_bins > 16384) return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    if (n == 0) return LC_MOE_OK;  // an empty idx may be a null pointer
    if (!idx) return LC_MOE_ERR_INVALID_ARG;
    if (!aligned16(idx) || !aligned16(ws)) return LC_MOE_ERR_MISALIGNED;
    LC_TRY(device_ok());
    LC_CUDA(launch_hist(idx, n, n_bins, counts, at<uint32_t>(ws, 0), static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_permute(const lc_moe_shape* s, const int32_t* idx, const void* x, int32_t* offsets,
                   int32_t* row_token, int32_t* pair_row, void* x_perm, void* ws, size_t ws_bytes,
                   void* stream) {
    LC_TRY(check_shape(s));
    if (!idx || !offsets || !row_token || !pair_row || !ws || (x_perm && !x))
        return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < permute_ws_bytes(s)) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    for (const void* p : {static_cast<const void*>(idx), x, static_cast<const void*>(x_perm),
                          static_cast<const void*>(ws)})
        if (p && !aligned16(p)) return LC_MOE_ERR_MISALIGNED;
    LC_TRY(device_ok());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    LC_CUDA(launch_permute(idx, s->T, s->K, s->N, s->N + s->Z, offsets, row_token, pair_row,
                           at<int32_t>(ws, kStatusBytes), at<uint32_t>(ws, 0), st));
    if (x_perm) LC_CUDA(launch_gather(x, s->T, s->d, s->K, pair_row, x_perm, at<uint32_t>(ws, 0), st));
    return LC_MOE_OK;
}

int lc_moe_expert_ffn(const lc_moe_shape* s, const void* x_perm, const int32_t* offsets,
                      const void* w13, const void* w2, void* h, void* y, void* ws,
                      size_t ws_bytes, void* stream) {
    LC_TRY(check_shape(s));
    if (!x_perm || !offsets || !w13 || !w2 || !h || !y || !ws) return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    for (const void* p : {x_perm, w13, w2, static_cast<const void*>(h), static_cast<const void*>(y),
                          static_cast<const void*>(ws)})
        if (!aligned16(p)) return LC_MOE_ERR_MISALIGNED;
    if (s->T == 0) return LC_MOE_OK;
    LC_TRY(device_ok());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    const int64_t rows_cap = static_cast<int64_t>(s->T) * s->K;
    uint32_t* status = at<uint32_t>(ws, 0);
    LC_CUDA(launch_grouped_swiglu(x_perm, rows_cap, offsets, s->N, w13, s->d, s->I, h, status, st));
    LC_CUDA(launch_grouped_down(h, rows_cap, offsets, s->N, w2, s->d, s->I, y, status, st));
    return LC_MOE_OK;
}

int lc_moe_combine(const lc_moe_shape* s, const void* x, const void* y, const float* gate,
                   const int32_t* pair_row, void* out, void* ws, size_t ws_bytes, void* stream) {
    LC_TRY(check_shape(s));
    if (!x || !y || !gate || !pair_row || !out || !ws) return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    for (const void* p : {x, y, static_cast<const void*>(out), static_cast<const void*>(ws)})
        if (!aligned16(p)) return LC_MOE_ERR_MISALIGNED;
    if (s->T == 0) return LC_MOE_OK;
    LC_TRY(device_ok());
    LC_CUDA(launch_combine(x, y, gate, pair_row, s->T, s->d, s->K, out, static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_ep_regroup_plan(const int32_t* cnt, int32_t G, int32_t n_local, int32_t* perm, int64_t m_cap,
                           int32_t* offsets, void* ws, size_t ws_bytes, void* stream) {
    if (!cnt || !offsets || !ws || (m_cap > 0 && !perm)) return LC_MOE_ERR_INVALID_ARG;
    if (G < 1 || n_local < 1 || m_cap < 0) return LC_MOE_ERR_INVALID_ARG;
    if (static_cast<int64_t>(G) * n_local > 2048 || m_cap >= (int64_t(1) << 31)) return LC_MOE_ERR_UNSUPPORTED_SHAPE;
    if (ws_bytes < kStatusBytes) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(ws)) return LC_MOE_ERR_MISALIGNED;
    LC_TRY(device_ok());
    LC_CUDA(launch_regroup_plan(cnt, G, n_local, perm, m_cap, offsets, at<uint32_t>(ws, 0),
                                static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_copy_rows(const void* src, void* dst, const int32_t* map, int64_t n, int32_t row_bytes,
                     int32_t scatter, void* ws, size_t ws_bytes, void* stream) {
    if (n < 0 || row_bytes <= 0 || row_bytes % 16 || (scatter != 0 && scatter != 1) || !ws)
        return LC_MOE_ERR_INVALID_ARG;
    if (n > 0 && (!src || !dst || !map)) return LC_MOE_ERR_INVALID_ARG;
    if (ws_bytes < kStatusBytes) return LC_MOE_ERR_WORKSPACE_TOO_SMALL;
    for (const void* p : {src, static_cast<const void*>(dst), static_cast<const void*>(ws)})
        if (p && !aligned16(p)) return LC_MOE_ERR_MISALIGNED;
    if (n == 0) return LC_MOE_OK;
    LC_TRY(device_ok());
    LC_CUDA(launch_copy_rows(src, dst, map, n, row_bytes, scatter, at<uint32_t>(ws, 0),
                             static_cast<cudaStream_t>(stream)));
    return LC_MOE_OK;
}

int lc_moe_permute_noalloc(const lc_moe_shape* s, const int32_t* idx, const void* x,
                           int32_t* offsets, int32_t* row_token, int32_t* pair_row, void* x_perm,
                           uint32_t* status, void* stream) {
    LC_TRY(check_shape(s));
    if (!idx || !offsets || !row_token || !pair_row || (x_perm && !x)) return LC_MOE_ERR_INVALID_ARG;
    if (!permute_noalloc_fits(s->T, s->N)) return LC_MOE_ERR_UNSUPPORTED_SHAPE;
    for (const void* p : {static_cast<const void*>(idx), x, static_cast<const void*>(x_perm)})
        if (p && !aligned16(p)) return LC_MOE_ERR_MISALIGNED;
    LC_TRY(device_ok());
    cudaStream_t st = static_cast<cudaStream_t>(stream);
    LC_CUDA(launch_permute_noalloc(idx, s->T, s->K, s->N, s->N + s->Z, offsets, row_token, pair_row,
                                   status, st));
    if (x_perm) LC_CUDA(launch_gather(x, s->T, s->d, s->K, pair_row, x_perm, status, st));
    return LC_MOE_OK;
}

}  // extern "C"

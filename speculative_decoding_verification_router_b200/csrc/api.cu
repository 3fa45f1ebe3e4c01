// Library-level entry points: device status word, bounded-wait limit and its
// self-test, launch tracing, the whole-layer composite, version/strings.
#include <stdio.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "ms_common.cuh"
#include "layer_fused.cuh"

namespace ms {

// implemented next to their kernels
ms_status rmsnorm_launch(const float*, const float*, int, int, float, void*, cudaStream_t);
ms_status route_launch(const void*, const float*, const float*, int, int, int, int, int, int32_t*,
                       float*, cudaStream_t);
ms_status route_cluster_launch(const void*, bool, float, const float*, const float*, int, int, int, int, int,
                               int32_t*, float*, void*, cudaStream_t);
size_t permute_ws_bytes(int, int, int);
ms_status permute_launch(const int32_t*, int, int, int, int32_t*, int32_t*, int32_t*, void*, int32_t*,
                         cudaStream_t);
size_t ffn_ws_bytes(int, int, int, int, int, int);
size_t route_tc_ws_bytes(int, int);
bool route_tc_supported(int, int, int);
ms_status route_tc_launch(const void*, const float*, const float*, int, int, int, int, int, int32_t*, float*, void*,
                          int32_t*, cudaStream_t);
ms_status ffn_launch(const void*, const int32_t*, const int32_t*, const void*, const void*, const void*,
                     const void*, int, int, int, int, int, int, void*, ms_dtype, float*, void*, cudaStream_t);
ms_status combine_launch(const void*, ms_dtype, const float*, const int32_t*, const float*, const float*,
                         int, int, int, float*, void*, cudaStream_t, bool);
void set_device_trace(void*);

static const char* kNames[K_COUNT] = {
    "rmsnorm",        "route_rows",      "route_tiled",     "route_cluster", "permute_count", "permute_scatter",
    "ffn_prep",       "gemm1_stream",    "gemm2_stream",    "gemm1_tiled",   "gemm2_tiled",  "ffn_finish",
    "lm_head_stream", "combine",         "verify_partial",  "verify_final",  "verify_cluster", "verify_keys", "wait_probe",
    "pack_weights",   "mtp_prep",        "moe_stream_layer", "route_tc",     "route_split"};

const char* kernel_name(int id) { return (id >= 0 && id < K_COUNT) ? kNames[id] : "?"; }

// ------------------------------------------------------------ errors
static thread_local char g_err[256] = "";
void set_cuda_error(cudaError_t e) {
    snprintf(g_err, sizeof g_err, "%s: %s", cudaGetErrorName(e), cudaGetErrorString(e));
}

// ------------------------------------------------------------ wait limit
static uint64_t g_wait_limit_ns = 1000000000ull;
uint64_t wait_limit_ns() { return g_wait_limit_ns; }

// ------------------------------------------------------------ batch-invariant schedules
static std::atomic<int> g_batch_invariant{0};
int batch_invariant() { return g_batch_invariant.load(std::memory_order_relaxed); }

// ------------------------------------------------------------ tracing
struct TraceRec {
    int id;
    cudaEvent_t start, stop;
};
static std::mutex g_trace_mu;
static std::vector<cudaEvent_t> g_events;   // pool: 2 per record
static std::vector<TraceRec> g_recs;
static int g_capacity = 0;
static bool g_trace_on = false;

// Inside stream capture an event must be recorded as an external record node,
// otherwise it only orders work within the capture and never gets a timestamp.
static void record(cudaEvent_t ev, cudaStream_t s) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    cudaStreamIsCapturing(s, &cs);
    cudaEventRecordWithFlags(ev, s, cs == cudaStreamCaptureStatusActive ? cudaEventRecordExternal
                                                                        : cudaEventRecordDefault);
}

void trace_mark(int id, cudaStream_t s, bool after) {
    if (!g_trace_on) return;
    std::lock_guard<std::mutex> lk(g_trace_mu);
    if (!after) {
        if (static_cast<int>(g_recs.size()) >= g_capacity) return;
        TraceRec r{id, g_events[2 * g_recs.size()], g_events[2 * g_recs.size() + 1]};
        record(r.start, s);
        g_recs.push_back(r);
    } else {
        if (g_recs.empty() || g_recs.back().id != id) return;
        // the matching stop is recorded once per start
        record(g_recs.back().stop, s);
    }
}

// ------------------------------------------------------------ wait probe
__global__ void wait_probe_kernel(const int32_t* flag, int32_t expect, int32_t* status, uint64_t limit_ns) {
    grid_dep_wait();
    grid_dep_launch();
    const uint64_t t0 = global_ns();
    for (uint32_t i = 0;; ++i) {
        if (*reinterpret_cast<const volatile int32_t*>(flag) == expect) {
            *status = MS_OK;
            return;
        }
        if ((i & 255u) == 0 && global_ns() - t0 > limit_ns) {
            *status = MS_ERR_TIMEOUT;
            return;
        }
    }
}

// ------------------------------------------------------------ layer composite
struct LayerWs {
    void* xhat;
    int32_t *idx, *offsets, *perm, *slot;
    float *w, *y_perm, *y_sh, *logits;
    void *perm_ws, *ffn_ws, *route_ws;
    size_t perm_bytes, ffn_bytes, bytes;
};

static LayerWs layer_layout(void* base, int T, int H, int E, int I, int S, int k) {
    LayerWs w{};
    char* p = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) -> char* {
        char* r = p ? p + off : nullptr;
        off += align_up(bytes > 0 ? bytes : 1, 1024);
        return r;
    };
    // the expert workspace first: its status word then sits at ws + 0
    w.ffn_bytes = ffn_ws_bytes(T, H, E, I, S, k);
    w.ffn_ws = take(w.ffn_bytes);
    w.xhat = take(static_cast<size_t>(T) * H * 2);
    w.idx = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
    w.w = reinterpret_cast<float*>(take(static_cast<size_t>(T) * k * 4));
    w.offsets = reinterpret_cast<int32_t*>(take(static_cast<size_t>(E + 1) * 4));
    w.perm = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
    w.slot = reinterpret_cast<int32_t*>(take(static_cast<size_t>(T) * k * 4));
    w.perm_bytes = permute_ws_bytes(T, k, E);
    w.perm_ws = take(w.perm_bytes);
    w.y_perm = reinterpret_cast<float*>(take(static_cast<size_t>(T) * k * H * (T <= 128 ? 4 : 2)));
    w.y_sh = reinterpret_cast<float*>(take(static_cast<size_t>(T) * H * 4));
    w.logits = reinterpret_cast<float*>(take(static_cast<size_t>(T) * E * 4));
    w.route_ws = T >= 1024 ? take(route_tc_ws_bytes(E, H)) : nullptr;   // the split router weights
    w.bytes = off;
    return w;
}

}  // namespace ms

extern "C" {

size_t moe_layer_workspace_size(int T, int H, int E, int I, int S, int k) {
    if (T <= 0 || H <= 0 || E <= 0 || I <= 0 || S < 0 || k <= 0) return 0;
    return ms::layer_layout(nullptr, T, H, E, I, S, k).bytes;
}

ms_status moe_layer_forward(const float* a, const float* w_router, const float* logit_bias,
                            const void* w_gate_up, const void* w_down, const void* ws_gate_up,
                            const void* ws_down, int T, int H, int E, int I, int S, int k, int renormalize,
                            float* out, void* ws, size_t ws_bytes, void* stream) {
    if (!a || !w_router || !w_gate_up || !w_down || !out) return MS_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || E <= 0 || I <= 0 || S < 0 || k <= 0 || k > E) return MS_ERR_INVALID_ARG;
    if (S > 0 && (!ws_gate_up || !ws_down)) return MS_ERR_INVALID_ARG;
    if (E > 256 || k > 32 || H % 128 != 0 || I % 128 != 0 || S > 8) return MS_ERR_UNSUPPORTED;
    if (T > 128 && H > 12288) return MS_ERR_UNSUPPORTED;   // the tiled path stages whole token rows
    const ms::LayerWs w = ms::layer_layout(ws, T, H, E, I, S, k);
    if (!ws || ws_bytes < w.bytes) return MS_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 1023u) return MS_ERR_INVALID_ARG;
    if (!ms::aligned16(a) || !ms::aligned16(out) || !ms::aligned16(w_router)) return MS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const ms_dtype ydt = T <= 128 ? MS_F32 : MS_BF16;
    int32_t* status = static_cast<int32_t*>(w.ffn_ws);
    // The status word reports this call's device-side conditions only; the
    // fused kernel's grid-barrier counter shares its 256-byte block.
    cudaError_t ce = cudaMemsetAsync(status, 0, 256, s);
    if (ce != cudaSuccess) {
        ms::set_cuda_error(ce);
        return MS_ERR_CUDA;
    }
    if (!ms::batch_invariant() && ms::layer_fused_supported(T, H, E, I, S, k)) {
        // verify-sized batch: the whole layer in one persistent kernel
        ms::LfBuffers b{};
        ms::ffn_ws_buffers(w.ffn_ws, T, H, E, I, S, k, b);
        b.logits = w.logits;
        b.y_perm = w.y_perm;
        b.y_sh = w.y_sh;
        b.idx = w.idx;
        b.off = w.offsets;
        b.perm = w.perm;
        b.slot = w.slot;
        b.w = w.w;
        b.bar = reinterpret_cast<unsigned int*>(static_cast<char*>(w.ffn_ws) + 128);
        return ms::layer_fused_launch(a, w_router, logit_bias, w_gate_up, w_down, ws_gate_up, ws_down, T, H, E, I, S,
                                      k, renormalize, 1e-6f, out, b, s);
    }
    ms_status st;
    if (T < 1024) {
        // normalisation fused into the router's clusters
        st = ms::route_cluster_launch(a, true, 1e-6f, w_router, logit_bias, T, H, E, k, renormalize, w.idx, w.w,
                                      w.xhat, s);
    } else {
        st = ms::rmsnorm_launch(a, nullptr, T, H, 1e-6f, w.xhat, s);
        // prefill-sized: the router on the tensor cores (B200: 281 -> ~20 us at
        // 36,992 tokens) where the shape allows, else the fp32 CUDA-core router
        if (st == MS_OK && ms::route_tc_supported(E, k, H))
            st = ms::route_tc_launch(w.xhat, w_router, logit_bias, T, H, E, k, renormalize, w.idx, w.w, w.route_ws,
                                     status, s);
        else if (st == MS_OK)
            st = ms::route_launch(w.xhat, w_router, logit_bias, T, H, E, k, renormalize, w.idx, w.w, s);
    }
    if (st == MS_OK) st = ms::permute_launch(w.idx, T, k, E, w.offsets, w.perm, w.slot, w.perm_ws, status, s);
    if (st == MS_OK)
        st = ms::ffn_launch(w.xhat, w.offsets, w.perm, w_gate_up, w_down, ws_gate_up, ws_down, T, H, E, I, S, k,
                            w.y_perm, ydt, S > 0 ? w.y_sh : nullptr, w.ffn_ws, s);
    if (st == MS_OK)
        // slots and gate weights (router, permute) and the residual are several
        // launches back: the combine may read them before its dependency wait
        st = ms::combine_launch(w.y_perm, ydt, S > 0 ? w.y_sh : nullptr, w.slot, w.w, a, T, H, k, out, nullptr, s,
                                true);
    return st;
}

ms_status ms_device_status(void* ws, void* stream) {
    if (!ws) return MS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t host = 0;
    cudaError_t e = cudaMemcpyAsync(&host, ws, sizeof host, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof host, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) {
        ms::set_cuda_error(e);
        return MS_ERR_CUDA;
    }
    return static_cast<ms_status>(host);
}

void ms_set_wait_limit_ns(uint64_t ns) { ms::g_wait_limit_ns = ns; }

void ms_set_batch_invariant(int on) { ms::g_batch_invariant.store(on ? 1 : 0, std::memory_order_relaxed); }
int ms_get_batch_invariant(void) { return ms::batch_invariant(); }

ms_status ms_set_device_trace(void* buf, size_t bytes) {
    if (buf && bytes < static_cast<size_t>(8) * 256 * 8 * sizeof(uint64_t)) return MS_ERR_WORKSPACE;
    ms::set_device_trace(buf);
    return MS_OK;
}
uint64_t ms_get_wait_limit_ns(void) { return ms::g_wait_limit_ns; }

ms_status ms_debug_bounded_wait(const int32_t* flag, int32_t expect, int32_t* status, void* stream) {
    if (!flag || !status) return MS_ERR_INVALID_ARG;
    return ms::launch(ms::K_WAIT_PROBE, ms::wait_probe_kernel, dim3(1), dim3(1), 0,
                      static_cast<cudaStream_t>(stream), flag, expect, status, ms::g_wait_limit_ns);
}

ms_status ms_trace_enable(int capacity) {
    if (capacity <= 0) return MS_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lk(ms::g_trace_mu);
    while (static_cast<int>(ms::g_events.size()) < 2 * capacity) {
        cudaEvent_t ev;
        cudaError_t e = cudaEventCreate(&ev);
        if (e != cudaSuccess) {
            ms::set_cuda_error(e);
            return MS_ERR_CUDA;
        }
        ms::g_events.push_back(ev);
    }
    ms::g_capacity = capacity;
    ms::g_recs.clear();
    ms::g_trace_on = true;
    return MS_OK;
}

void ms_trace_disable(void) { ms::g_trace_on = false; }

void ms_trace_reset(void) {
    std::lock_guard<std::mutex> lk(ms::g_trace_mu);
    ms::g_recs.clear();
}

int ms_trace_count(void) {
    std::lock_guard<std::mutex> lk(ms::g_trace_mu);
    return static_cast<int>(ms::g_recs.size());
}

ms_status ms_trace_read(int i, const char** kernel_name, float* ms_out) {
    std::lock_guard<std::mutex> lk(ms::g_trace_mu);
    if (i < 0 || i >= static_cast<int>(ms::g_recs.size()) || !ms_out) return MS_ERR_INVALID_ARG;
    const ms::TraceRec& r = ms::g_recs[i];
    if (kernel_name) *kernel_name = ms::kernel_name(r.id);
    cudaError_t e = cudaEventElapsedTime(ms_out, r.start, r.stop);
    if (e != cudaSuccess) {
        ms::set_cuda_error(e);
        return MS_ERR_CUDA;
    }
    return MS_OK;
}

const char* ms_status_string(ms_status s) {
    switch (s) {
        case MS_OK: return "ok";
        case MS_ERR_INVALID_ARG: return "invalid argument";
        case MS_ERR_UNSUPPORTED: return "unsupported shape";
        case MS_ERR_WORKSPACE: return "workspace missing or too small";
        case MS_ERR_CUDA: return "CUDA error";
        case MS_ERR_TIMEOUT: return "device-side bounded wait timed out";
        case MS_ERR_DEVICE_INDEX: return "device-side index out of range";
        case MS_ERR_DRAIN_TIMEOUT: return "device-side drain after a timeout ran out (device state undefined)";
    }
    return "unknown status";
}

const char* ms_last_cuda_error_string(void) { return ms::g_err; }

int ms_version(void) { return 100; }

}  // extern "C"

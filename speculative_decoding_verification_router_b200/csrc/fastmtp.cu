// FastMTP draft block on the device: one dense block applied K times with
// shared weights, each step fed the previous step's hidden state and token
// (jina.ai, "Modèle et entraînement"; the d9249 blog's component table).
//
// The pages do not describe the block's inside; this is the multi-token-
// prediction module of the decoder family it extends, without attention:
//   x  = [bf16(RMSNorm(h)); bf16(RMSNorm(emb[t]))]          (2H)
//   u  = W_proj x                                            (H)
//   h' = u + SwiGLU(bf16(RMSNorm(u)))                        (dense, intermediate I)
//   t' = argmax_v bf16(W_lm bf16(RMSNorm(h')))                (the verifier's vocab head)
// Every step is built from the library's own kernels: a prep kernel (token
// embedding gather + both norms into the concatenated operand), the
// streaming GEMM as a linear layer, the expert FFN with one dense expert, the
// combine kernel for the residual, and the vocab head with the argmax in its
// epilogue.
#include "ms_common.cuh"

namespace ms {

// offsets, perm, slot and weight arrays of a one-group, identity-order FFN
__global__ void __launch_bounds__(128) mtp_setup_kernel(int B, int32_t* offsets, int32_t* perm, int32_t* slot,
                                                        float* w1) {
    grid_dep_wait();
    grid_dep_launch();
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x) {
        perm[b] = b;
        slot[b] = b;
        w1[b] = 1.f;
    }
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        offsets[0] = 0;
        offsets[1] = B;
    }
}

// One warp per row b < rows_pad.  Rows b < B: x[b] = [bf16(RMSNorm(h[b])),
// bf16(RMSNorm(emb[tok[b]]))] (fp32 sums of squares, IEEE sqrt and divide);
// rows B.. are zero.  With drafts set, also drafts[b*K + col] = tok[b] (the
// previous step's draft token).  A token outside [0, V) is flagged and its
// embedding taken as zero.
__global__ void __launch_bounds__(256) mtp_prep_kernel(const float* __restrict__ h, const int32_t* __restrict__ tok,
                                                       const __nv_bfloat16* __restrict__ emb, int B, int H, int V,
                                                       int rows_pad, float eps, __nv_bfloat16* __restrict__ x,
                                                       int32_t* __restrict__ drafts, int K, int col,
                                                       int32_t* status) {
    grid_dep_wait();
    grid_dep_launch();
    const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (b >= rows_pad) return;
    __nv_bfloat162* xr = reinterpret_cast<__nv_bfloat162*>(x + static_cast<size_t>(b) * 2 * H);
    const int n4 = H >> 2;
    if (b >= B) {
        for (int i = lane; i < H; i += 32) xr[i] = __floats2bfloat162_rn(0.f, 0.f);
        return;
    }
    int t = __ldg(tok + b);
    if (drafts && lane == 0) drafts[static_cast<size_t>(b) * K + col] = t;
    const bool tok_ok = t >= 0 && t < V;
    if (!tok_ok) {
        if (lane == 0) report_status(status, MS_ERR_DEVICE_INDEX);
        t = 0;
    }
    // hidden state half
    const float4* hr = reinterpret_cast<const float4*>(h + static_cast<size_t>(b) * H);
    float ss = 0.f;
    for (int i = lane; i < n4; i += 32) {
        const float4 v = __ldg(hr + i);
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
    for (int i = lane; i < n4; i += 32) {
        const float4 v = __ldg(hr + i);
        xr[2 * i] = __floats2bfloat162_rn(v.x * inv, v.y * inv);
        xr[2 * i + 1] = __floats2bfloat162_rn(v.z * inv, v.w * inv);
    }
    // token embedding half (bf16 row, widened exactly)
    const __nv_bfloat162* er = reinterpret_cast<const __nv_bfloat162*>(emb + static_cast<size_t>(t) * H);
    const int n2 = H >> 1;
    ss = 0.f;
    for (int i = lane; i < n2; i += 32) {
        const float2 v = tok_ok ? __bfloat1622float2(er[i]) : make_float2(0.f, 0.f);
        ss += v.x * v.x + v.y * v.y;
    }
    ss = warp_sum(ss);
    inv = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
    for (int i = lane; i < n2; i += 32) {
        const float2 v = tok_ok ? __bfloat1622float2(er[i]) : make_float2(0.f, 0.f);
        xr[n2 + i] = __floats2bfloat162_rn(v.x * inv, v.y * inv);
    }
}

__global__ void __launch_bounds__(128) mtp_collect_kernel(const int32_t* __restrict__ tok, int B, int K, int col,
                                                          int32_t* __restrict__ drafts) {
    grid_dep_wait();
    grid_dep_launch();
    for (int b = blockIdx.x * blockDim.x + threadIdx.x; b < B; b += gridDim.x * blockDim.x)
        drafts[static_cast<size_t>(b) * K + col] = tok[b];
}

// implemented next to their kernels
size_t ffn_ws_bytes(int, int, int, int, int, int);
ms_status ffn_launch(const void*, const int32_t*, const int32_t*, const void*, const void*, const void*,
                     const void*, int, int, int, int, int, int, void*, ms_dtype, float*, void*, cudaStream_t);
size_t lm_ws_bytes(int, int);
ms_status lm_launch(const void*, const void*, int, int, int, void*, void*, cudaStream_t, unsigned long long*,
                    int32_t*);
size_t linear_ws_bytes(int);
ms_status linear_launch(const void*, int, int, int, const void*, int, const int32_t*, float*, void*, int32_t*,
                        cudaStream_t);
ms_status rmsnorm_launch(const float*, const float*, int, int, float, void*, cudaStream_t);
ms_status combine_launch(const void*, ms_dtype, const float*, const int32_t*, const float*, const float*, int,
                         int, int, float*, void*, cudaStream_t, bool);
ms_status verify_keys_launch(const unsigned long long*, int, int, int, const int32_t*, int32_t*, int32_t*,
                             int32_t*, cudaStream_t);

struct MtpWs {
    void *ffn, *lm, *lin;
    __nv_bfloat16 *xcat, *xh;
    float *u, *y, *h[2], *w1;
    int32_t *tok[2], *offsets, *perm, *slot, *ctmp, *ntmp;
    unsigned long long* keys;
    int rows_pad;
    size_t bytes;
};

static MtpWs mtp_layout(void* base, int B, int H, int I, int V) {
    MtpWs w{};
    char* p = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) -> char* {
        char* r = p ? p + off : nullptr;
        off += align_up(bytes > 0 ? bytes : 1, 1024);
        return r;
    };
    w.rows_pad = static_cast<int>(align_up(B, 128));
    w.ffn = take(ffn_ws_bytes(B, H, 1, I, 0, 1));   // first: its status word is ws + 0
    w.lm = take(lm_ws_bytes(H, V));
    w.lin = take(linear_ws_bytes(B));
    w.xcat = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(w.rows_pad) * 2 * H * 2));
    w.xh = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(B) * H * 2));
    w.u = reinterpret_cast<float*>(take(static_cast<size_t>(B) * H * 4));
    w.y = reinterpret_cast<float*>(take(static_cast<size_t>(B) * H * 4));
    w.h[0] = reinterpret_cast<float*>(take(static_cast<size_t>(B) * H * 4));
    w.h[1] = reinterpret_cast<float*>(take(static_cast<size_t>(B) * H * 4));
    w.tok[0] = reinterpret_cast<int32_t*>(take(static_cast<size_t>(B) * 4));
    w.tok[1] = reinterpret_cast<int32_t*>(take(static_cast<size_t>(B) * 4));
    w.offsets = reinterpret_cast<int32_t*>(take(8));
    w.perm = reinterpret_cast<int32_t*>(take(static_cast<size_t>(B) * 4));
    w.slot = reinterpret_cast<int32_t*>(take(static_cast<size_t>(B) * 4));
    w.w1 = reinterpret_cast<float*>(take(static_cast<size_t>(B) * 4));
    w.ctmp = reinterpret_cast<int32_t*>(take(static_cast<size_t>(B) * 4));
    w.ntmp = reinterpret_cast<int32_t*>(take(static_cast<size_t>(B) * 4));
    w.keys = reinterpret_cast<unsigned long long*>(take(static_cast<size_t>(B) * (V / 16) * 8));
    w.bytes = off;
    return w;
}

}  // namespace ms

extern "C" size_t fastmtp_draft_workspace_size(int B, int H, int I, int V) {
    if (B <= 0 || H <= 0 || I <= 0 || V <= 0) return 0;
    return ms::mtp_layout(nullptr, B, H, I, V).bytes;
}

extern "C" ms_status fastmtp_draft(const float* h0, const int32_t* tok0, const void* emb, const void* w_proj,
                                   const void* w_gate_up, const void* w_down, const void* w_lm, int B, int H,
                                   int I, int V, int K, int32_t* drafts, float* h_out, void* ws, size_t ws_bytes,
                                   void* stream) {
    if (!h0 || !tok0 || !emb || !w_proj || !w_gate_up || !w_down || !w_lm || !drafts) return MS_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || I <= 0 || V <= 0 || K <= 0) return MS_ERR_INVALID_ARG;
    if (B > 128 || K > 8 || H % 128 != 0 || I % 128 != 0 || V % 128 != 0 || V > (1 << 30))
        return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(h0) || !ms::aligned16(emb) || !ms::aligned16(w_proj) || !ms::aligned16(w_gate_up) ||
        !ms::aligned16(w_down) || !ms::aligned16(w_lm) || (h_out && !ms::aligned16(h_out)))
        return MS_ERR_INVALID_ARG;
    const ms::MtpWs w = ms::mtp_layout(ws, B, H, I, V);
    if (!ws || ws_bytes < w.bytes) return MS_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 1023u) return MS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    int32_t* status = static_cast<int32_t*>(ws);
    cudaError_t ce = cudaMemsetAsync(status, 0, sizeof(int32_t), s);
    if (ce != cudaSuccess) {
        ms::set_cuda_error(ce);
        return MS_ERR_CUDA;
    }
    const float eps = 1e-6f;
    ms_status st = ms::launch(ms::K_MTP_PREP, ms::mtp_setup_kernel, dim3(1), dim3(128), 0, s, B, w.offsets, w.perm,
                              w.slot, w.w1);
    const float* h_cur = h0;
    const int32_t* t_cur = tok0;
    for (int i = 0; i < K && st == MS_OK; ++i) {
        float* h_next = (i == K - 1 && h_out) ? h_out : w.h[i & 1];
        int32_t* t_next = w.tok[i & 1];
        const int rows_per_block = 8;
        st = ms::launch(ms::K_MTP_PREP, ms::mtp_prep_kernel, dim3((w.rows_pad + rows_per_block - 1) / rows_per_block),
                        dim3(256), 0, s, h_cur, t_cur, static_cast<const __nv_bfloat16*>(emb), B, H, V, w.rows_pad,
                        eps, w.xcat, i > 0 ? drafts : static_cast<int32_t*>(nullptr), K, i - 1, status);
        if (st == MS_OK)
            st = ms::linear_launch(w.xcat, w.rows_pad, B, 2 * H, w_proj, H, w.offsets, w.u, w.lin, status, s);
        if (st == MS_OK) st = ms::rmsnorm_launch(w.u, nullptr, B, H, eps, w.xh, s);
        if (st == MS_OK)
            st = ms::ffn_launch(w.xh, w.offsets, w.perm, w_gate_up, w_down, nullptr, nullptr, B, H, 1, I, 0, 1, w.y,
                                MS_F32, nullptr, w.ffn, s);
        if (st == MS_OK)
            st = ms::combine_launch(w.y, MS_F32, nullptr, w.slot, w.w1, w.u, B, H, 1, h_next, nullptr, s, false);
        if (st == MS_OK) st = ms::rmsnorm_launch(h_next, nullptr, B, H, eps, w.xh, s);
        if (st == MS_OK) st = ms::lm_launch(w.xh, w_lm, B, H, V, nullptr, w.lm, s, w.keys, status);
        if (st == MS_OK)
            st = ms::verify_keys_launch(w.keys, V / 16, B, 0, nullptr, t_next, w.ctmp, w.ntmp, s);
        h_cur = h_next;
        t_cur = t_next;
    }
    if (st == MS_OK)
        st = ms::launch(ms::K_MTP_PREP, ms::mtp_collect_kernel, dim3((B + 127) / 128), dim3(128), 0, s, t_cur, B, K,
                        K - 1, drafts);
    return st;
}

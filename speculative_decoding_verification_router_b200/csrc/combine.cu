// a4: gate-weighted un-permute of the routed expert outputs, plus the shared
// experts and the residual: out = sum_j w_j * y[slot_j] + y_shared + residual.
#include "ms_common.cuh"

namespace ms {

__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}

__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(q[i] << 16);
        v[2 * i + 1] = __uint_as_float(q[i] & 0xffff0000u);
    }
}

// One thread per 8 consecutive hidden elements of one token (grid-stride).
// With `early` set (the layer's own chain, where the slots, gate weights and
// residual were written two or more launches back), a thread reads those of
// its first element before waiting on the previous kernel, leaving only the
// expert outputs' round trip after the wait.
constexpr int CB_KPRE = 8;

template <typename TY>
__global__ void __launch_bounds__(256) combine_kernel(const TY* __restrict__ y,
                                                      const float* __restrict__ ysh,
                                                      const int32_t* __restrict__ slot,
                                                      const float* __restrict__ w,
                                                      const float* __restrict__ res, int T, int H,
                                                      int k, float* __restrict__ out,
                                                      __nv_bfloat16* __restrict__ out_bf16, int early) {
    const int n8 = H >> 3;
    const long total = static_cast<long>(T) * n8;
    const long rows = static_cast<long>(T) * k;
    const long v0 = blockIdx.x * static_cast<long>(blockDim.x) + threadIdx.x;
    const bool pre = early && k <= CB_KPRE && v0 < total;
    int pr[CB_KPRE];
    float pw[CB_KPRE], prv[8];
    if (pre) {
        const int t = static_cast<int>(v0 / n8);
#pragma unroll
        for (int j = 0; j < CB_KPRE; ++j)
            if (j < k) {
                pr[j] = __ldg(slot + static_cast<size_t>(t) * k + j);
                pw[j] = __ldg(w + static_cast<size_t>(t) * k + j);
            }
        if (res) load8(res + static_cast<size_t>(t) * H + static_cast<int>(v0 % n8) * 8, prv);
    }
    grid_dep_wait();
    grid_dep_launch();
    for (long v = v0; v < total; v += static_cast<long>(gridDim.x) * blockDim.x) {
        const int t = static_cast<int>(v / n8);
        const int c = static_cast<int>(v % n8) * 8;
        const bool first = pre && v == v0;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        if (first) {
#pragma unroll
            for (int j = 0; j < CB_KPRE; ++j) {
                if (j >= k || pr[j] < 0 || pr[j] >= rows) continue;
                float yv[8];
                load8(y + static_cast<size_t>(pr[j]) * H + c, yv);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = fmaf(pw[j], yv[q], acc[q]);
            }
        } else {
            for (int j = 0; j < k; ++j) {
                const int r = __ldg(slot + static_cast<size_t>(t) * k + j);
                if (r < 0 || r >= rows) continue;
                const float wj = __ldg(w + static_cast<size_t>(t) * k + j);
                float yv[8];
                load8(y + static_cast<size_t>(r) * H + c, yv);
#pragma unroll
                for (int q = 0; q < 8; ++q) acc[q] = fmaf(wj, yv[q], acc[q]);
            }
        }
        const size_t o = static_cast<size_t>(t) * H + c;
        if (ysh) {
            float sv[8];
            load8(ysh + o, sv);
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] += sv[q];
        }
        if (res) {
            float rv[8];
            if (first) {
#pragma unroll
                for (int q = 0; q < 8; ++q) rv[q] = prv[q];
            } else {
                load8(res + o, rv);
            }
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] += rv[q];
        }
        float4* op = reinterpret_cast<float4*>(out + o);
        op[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
        op[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
        if (out_bf16) {
            __nv_bfloat162 b[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) b[q] = __floats2bfloat162_rn(acc[2 * q], acc[2 * q + 1]);
            *reinterpret_cast<uint4*>(out_bf16 + o) = *reinterpret_cast<uint4*>(b);
        }
    }
}

ms_status combine_launch(const void* y, ms_dtype ydt, const float* ysh, const int32_t* slot,
                         const float* w, const float* res, int T, int H, int k, float* out,
                         void* out_bf16, cudaStream_t s, bool early) {
    const long total = static_cast<long>(T) * (H / 8);
    const long want = (total + 255) / 256;
    const int grid = static_cast<int>(want < 8L * num_sms() ? want : 8L * num_sms());
    auto* ob = reinterpret_cast<__nv_bfloat16*>(out_bf16);
    if (ydt == MS_BF16)
        return launch(K_COMBINE, combine_kernel<__nv_bfloat16>, dim3(grid), dim3(256), 0, s,
                      reinterpret_cast<const __nv_bfloat16*>(y), ysh, slot, w, res, T, H, k, out, ob, early ? 1 : 0);
    return launch(K_COMBINE, combine_kernel<float>, dim3(grid), dim3(256), 0, s,
                  reinterpret_cast<const float*>(y), ysh, slot, w, res, T, H, k, out, ob, early ? 1 : 0);
}

}  // namespace ms

extern "C" ms_status moe_combine(const void* y_perm, ms_dtype y_perm_dtype, const float* y_shared,
                                 const int32_t* slot_of, const float* topk_w,
                                 const float* residual, int T, int H, int k, float* out,
                                 void* out_bf16, void* stream) {
    if (!y_perm || !slot_of || !topk_w || !out) return MS_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || k <= 0) return MS_ERR_INVALID_ARG;
    if (y_perm_dtype != MS_F32 && y_perm_dtype != MS_BF16) return MS_ERR_INVALID_ARG;
    if (H % 8 != 0) return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(y_perm) || !ms::aligned16(out) || (y_shared && !ms::aligned16(y_shared)) ||
        (residual && !ms::aligned16(residual)) || (out_bf16 && !ms::aligned16(out_bf16)))
        return MS_ERR_INVALID_ARG;
    return ms::combine_launch(y_perm, y_perm_dtype, y_shared, slot_of, topk_w, residual, T, H, k,
                              out, out_bf16, static_cast<cudaStream_t>(stream), false);
}

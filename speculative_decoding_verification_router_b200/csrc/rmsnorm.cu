// a0: RMSNorm of the residual stream into the bf16 expert input.
#include "ms_common.cuh"

namespace ms {

// One warp per row; float4 loads, fp32 sum of squares, IEEE sqrt/div.  Up to
// RN_KEEP float4 per lane (H <= 2,048) the row stays in registers between the
// two passes, all of its loads issued at once; longer rows are read twice.
constexpr int RN_KEEP = 16;

__global__ void __launch_bounds__(256) rmsnorm_kernel(const float* __restrict__ a,
                                                      const float* __restrict__ gamma, int T,
                                                      int H, float eps,
                                                      __nv_bfloat16* __restrict__ out) {
    grid_dep_wait();
    grid_dep_launch();
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (warp >= T) return;
    const float4* row = reinterpret_cast<const float4*>(a + static_cast<size_t>(warp) * H);
    const int n4 = H >> 2;
    __nv_bfloat162* orow = reinterpret_cast<__nv_bfloat162*>(out + static_cast<size_t>(warp) * H);
    const float4* g4 = reinterpret_cast<const float4*>(gamma);
    if (n4 <= 32 * RN_KEEP) {
        float4 v[RN_KEEP];
#pragma unroll
        for (int j = 0; j < RN_KEEP; ++j) {
            const int i = lane + 32 * j;
            v[j] = i < n4 ? __ldg(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < RN_KEEP; ++j) ss += v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
        ss = warp_sum(ss);
        const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
#pragma unroll
        for (int j = 0; j < RN_KEEP; ++j) {
            const int i = lane + 32 * j;
            if (i < n4) {
                const float4 g = gamma ? __ldg(g4 + i) : make_float4(1.f, 1.f, 1.f, 1.f);
                orow[2 * i] = __floats2bfloat162_rn(v[j].x * inv * g.x, v[j].y * inv * g.y);
                orow[2 * i + 1] = __floats2bfloat162_rn(v[j].z * inv * g.z, v[j].w * inv * g.w);
            }
        }
        return;
    }
    float ss = 0.f;
    for (int i = lane; i < n4; i += 32) {
        float4 v = __ldg(row + i);
        ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
    }
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + eps);
    for (int i = lane; i < n4; i += 32) {
        float4 v = __ldg(row + i);
        float4 g = gamma ? __ldg(g4 + i) : make_float4(1.f, 1.f, 1.f, 1.f);
        orow[2 * i] = __floats2bfloat162_rn(v.x * inv * g.x, v.y * inv * g.y);
        orow[2 * i + 1] = __floats2bfloat162_rn(v.z * inv * g.z, v.w * inv * g.w);
    }
}

ms_status rmsnorm_launch(const float* a, const float* gamma, int T, int H, float eps, void* out,
                         cudaStream_t s) {
    const int rows_per_block = 8;
    dim3 grid((T + rows_per_block - 1) / rows_per_block);
    return launch(K_RMSNORM, rmsnorm_kernel, grid, dim3(256), 0, s, a, gamma, T, H, eps,
                  reinterpret_cast<__nv_bfloat16*>(out));
}

}  // namespace ms

extern "C" ms_status moe_rmsnorm(const float* a, const float* gamma, int T, int H, float eps,
                                 void* xhat_bf16, void* stream) {
    if (!a || !xhat_bf16 || T <= 0 || H <= 0 || !(eps >= 0.f)) return MS_ERR_INVALID_ARG;
    if (H % 8 != 0) return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(a) || !ms::aligned16(xhat_bf16) || (gamma && !ms::aligned16(gamma)))
        return MS_ERR_INVALID_ARG;
    return ms::rmsnorm_launch(a, gamma, T, H, eps, xhat_bf16, static_cast<cudaStream_t>(stream));
}

// a1: router logits (fp32), softmax over all experts and top-k selection.
//
// Top-6 of 64 routed experts (clawpit.io, "Lean architecture with a
// compressed encoder").  Selection order: larger logit first, equal logits
// to the lower expert index.  Gate weight = softmax probability of the
// chosen expert (optionally renormalised over the k chosen).
#include <math.h>

#include "ms_common.cuh"

namespace ms {

constexpr int kMaxExperts = 256;

// One warp: softmax over z[0..E) and the k best experts, written to
// idx_out[0..k) / w_out[0..k).  Each lane holds experts lane, lane+32, ...
__device__ void warp_topk_softmax(const float* z, int E, int k, int renorm, int32_t* idx_out,
                                  float* w_out, int lane) {
    constexpr int kPer = kMaxExperts / 32;
    float v[kPer];
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < kPer; ++i) {
        const int e = lane + 32 * i;
        v[i] = e < E ? z[e] : -INFINITY;
        m = fmaxf(m, v[i]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        if (lane + 32 * i < E) s += expf(v[i] - m);
    s = warp_sum(s);
    uint32_t taken = 0;
    float wsum = 0.f;
    float wsel = 0.f;
    for (int j = 0; j < k; ++j) {
        float bv = -INFINITY;
        int bi = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < kPer; ++i) {
            const int e = lane + 32 * i;
            if (e < E && !((taken >> i) & 1u)) argmax_merge(bv, bi, v[i], e);
        }
        warp_argmax(bv, bi);
        if ((bi & 31) == lane) taken |= 1u << (bi >> 5);
        const float p = expf(bv - m) / s;
        wsum += p;
        if (lane == j) wsel = p;
        if (lane == 0) idx_out[j] = bi;
    }
    if (lane < k) w_out[lane] = renorm ? wsel / wsum : wsel;
}

// Small T: one block per token, 8 warps stride over experts; W_r rows are
// read with float4 loads (L2-resident after the first token).
__global__ void __launch_bounds__(256) route_rows_kernel(const __nv_bfloat16* __restrict__ x,
                                                         const float* __restrict__ wr,
                                                         const float* __restrict__ bias, int T,
                                                         int H, int E, int k, int renorm,
                                                         int32_t* __restrict__ idx,
                                                         float* __restrict__ w) {
    extern __shared__ float smem[];
    float* xs = smem;       // [H]
    float* z = smem + H;    // [E]
    grid_dep_wait();
    grid_dep_launch();
    const int t = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const uint4* xr = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H);
    for (int i = threadIdx.x; i < H / 8; i += blockDim.x) {
        uint4 u = __ldg(xr + i);
        const uint32_t p[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            xs[8 * i + 2 * q] = __uint_as_float(p[q] << 16);
            xs[8 * i + 2 * q + 1] = __uint_as_float(p[q] & 0xffff0000u);
        }
    }
    __syncthreads();
    for (int e = warp; e < E; e += blockDim.x / 32) {
        const float4* wrow = reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * H);
        float acc = 0.f;
        for (int h4 = lane; h4 < H / 4; h4 += 32) {
            float4 a = __ldg(wrow + h4);
            float4 b = *reinterpret_cast<const float4*>(xs + 4 * h4);
            acc = fmaf(a.x, b.x, acc);
            acc = fmaf(a.y, b.y, acc);
            acc = fmaf(a.z, b.z, acc);
            acc = fmaf(a.w, b.w, acc);
        }
        acc = warp_sum(acc);
        if (lane == 0) z[e] = bias ? acc + __ldg(bias + static_cast<size_t>(t) * E + e) : acc;
    }
    __syncthreads();
    if (warp == 0)
        warp_topk_softmax(z, E, k, renorm, idx + static_cast<size_t>(t) * k,
                          w + static_cast<size_t>(t) * k, lane);
}

// Large T (E <= 64): 128 tokens x 64 experts per block of 256 threads, an
// 8 x 4 register tile per thread, H walked in chunks of 32 through shared
// memory (stored transposed, k-major, with the next chunk's global loads
// issued before the current chunk's FMAs); then top-k per token from the
// logits, kept in the same shared memory.  fp32 FMAs in a fixed order.
constexpr int RT_TOK = 128, RT_EXP = 64, RT_K = 32;
constexpr int RT_XS = RT_TOK + 4, RT_WS = RT_EXP + 4;   // padded rows: conflict-free stores and loads

struct RouteTiledSmem {
    union {
        struct {
            float xs[RT_K][RT_XS];
            float ws[RT_K][RT_WS];
        } in;
        float zs[RT_TOK][RT_EXP + 1];
    };
};

__global__ void __launch_bounds__(256) route_tiled_kernel(const __nv_bfloat16* __restrict__ x,
                                                          const float* __restrict__ wr,
                                                          const float* __restrict__ bias, int T,
                                                          int H, int E, int k, int renorm,
                                                          int32_t* __restrict__ idx,
                                                          float* __restrict__ w) {
    __shared__ __align__(16) RouteTiledSmem sm;
    grid_dep_wait();
    grid_dep_launch();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int t0 = blockIdx.x * RT_TOK;
    const int ty = tid >> 4, tx = tid & 15;   // tokens ty*8.., experts tx*4..
    float acc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;

    // loader mapping: a warp covers 32 consecutive tokens (experts) of one
    // 8-wide (4-wide) h segment, so the transposed stores hit 32 banks
    const int xt = (tid & 31) + 32 * ((tid >> 5) >> 2);   // token 0..63 (+64 for the second load)
    const int xseg = (tid >> 5) & 3;                       // 8 h each
    const int we = tid & 63;                               // expert
    const int wseg = tid >> 6;                             // 4 h each, 0..3 (+4 for the second load)
    uint4 xr[2];
    float4 wv[2];
    auto fetch = [&](int h0) {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int t = t0 + xt + 64 * i;
            xr[i] = t < T ? __ldg(reinterpret_cast<const uint4*>(x + static_cast<size_t>(t) * H + h0 + xseg * 8))
                          : make_uint4(0, 0, 0, 0);
            wv[i] = we < E ? __ldg(reinterpret_cast<const float4*>(wr + static_cast<size_t>(we) * H + h0 +
                                                                    (wseg + 4 * i) * 4))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    };
    auto stash = [&]() {
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const uint32_t pq[4] = {xr[i].x, xr[i].y, xr[i].z, xr[i].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                sm.in.xs[xseg * 8 + 2 * q][xt + 64 * i] = __uint_as_float(pq[q] << 16);
                sm.in.xs[xseg * 8 + 2 * q + 1][xt + 64 * i] = __uint_as_float(pq[q] & 0xffff0000u);
            }
            const int hb = (wseg + 4 * i) * 4;
            sm.in.ws[hb + 0][we] = wv[i].x;
            sm.in.ws[hb + 1][we] = wv[i].y;
            sm.in.ws[hb + 2][we] = wv[i].z;
            sm.in.ws[hb + 3][we] = wv[i].w;
        }
    };
    fetch(0);
    for (int h0 = 0; h0 < H; h0 += RT_K) {
        stash();
        __syncthreads();
        if (h0 + RT_K < H) fetch(h0 + RT_K);   // in flight during the FMAs below
        // operands of step kk + 1 are read from shared memory while step kk's
        // 32 FMAs run (few warps per SM: the load latency must hide in ILP)
        float4 a0 = *reinterpret_cast<const float4*>(&sm.in.xs[0][ty * 8]);
        float4 a1 = *reinterpret_cast<const float4*>(&sm.in.xs[0][ty * 8 + 4]);
        float4 b = *reinterpret_cast<const float4*>(&sm.in.ws[0][tx * 4]);
#pragma unroll
        for (int kk = 0; kk < RT_K; ++kk) {
            float4 na0 = a0, na1 = a1, nb = b;
            if (kk + 1 < RT_K) {
                na0 = *reinterpret_cast<const float4*>(&sm.in.xs[kk + 1][ty * 8]);
                na1 = *reinterpret_cast<const float4*>(&sm.in.xs[kk + 1][ty * 8 + 4]);
                nb = *reinterpret_cast<const float4*>(&sm.in.ws[kk + 1][tx * 4]);
            }
            const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float bv[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 8; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
            a0 = na0;
            a1 = na1;
            b = nb;
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int t = t0 + ty * 8 + i, e = tx * 4 + j;
            float zv = acc[i][j];
            if (bias && t < T && e < E) zv += __ldg(bias + static_cast<size_t>(t) * E + e);
            sm.zs[ty * 8 + i][e] = zv;
        }
    __syncthreads();
    for (int r = warp; r < RT_TOK; r += 8) {
        const int t = t0 + r;
        if (t >= T) break;
        warp_topk_softmax(sm.zs[r], E, k, renorm, idx + static_cast<size_t>(t) * k,
                          w + static_cast<size_t>(t) * k, lane);
    }
}

// Small T: one cluster of RC_CTAS CTAs per TPC tokens.  CTA r computes the
// logits of experts [r*E/RC_CTAS, (r+1)*E/RC_CTAS) for the cluster's tokens --
// one warp per expert, whose W_r row is read once (float4 loads) and used for
// every token -- and stores them into CTA 0's shared memory (distributed
// shared memory); after the cluster barrier CTA 0 runs the softmax and top-k,
// one warp per token.  With NORM the CTAs first RMS-normalise the fp32
// residual rows themselves (eps, unit gain) and CTA 0 writes the bf16 result,
// so the layer needs no separate normalisation kernel.  Each token's logits
// are summed in the same order whatever TPC is.
constexpr int RC_CTAS = 8;
constexpr int RC_WPRE = 12;   // float4 of a router row per lane kept in registers (H <= 1536)

template <bool NORM, int TPC>
__global__ void __launch_bounds__(256) route_cluster_kernel(const void* __restrict__ xin,
                                                            const float* __restrict__ wr,
                                                            const float* __restrict__ bias, int T, int H,
                                                            int E, int k, int renorm, float eps,
                                                            int32_t* __restrict__ idx, float* __restrict__ w,
                                                            __nv_bfloat16* __restrict__ xhat_out) {
    extern __shared__ float smem[];
    float* xs = smem;            // [TPC][H] the tokens' normalised activations (bf16 values)
    float* z = smem + TPC * H;   // [TPC][E] logits, filled by every CTA of the cluster
    __shared__ float red[TPC][8];
    const uint32_t rank = cluster_rank();
    const int t0 = static_cast<int>(blockIdx.y) * TPC;
    const int nt = T - t0 < TPC ? T - t0 : TPC;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int per = (E + RC_CTAS - 1) / RC_CTAS;
    const int e0 = static_cast<int>(rank) * per;
    const int e1 = e0 + per < E ? e0 + per : E;
    // this warp's first router row, loaded before the dependency wait when it
    // fits the registers: no kernel of this library writes the router weights,
    // and a kernel of any other origin has completed before this one starts
    const bool wpre = H / 4 <= 32 * RC_WPRE && e0 + warp < e1;
    float4 wv[RC_WPRE];
    if (wpre) {
        const float4* wrow = reinterpret_cast<const float4*>(wr + static_cast<size_t>(e0 + warp) * H);
#pragma unroll
        for (int j = 0; j < RC_WPRE; ++j) {
            const int h4 = lane + 32 * j;
            wv[j] = h4 < H / 4 ? __ldg(wrow + h4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
    }
    grid_dep_wait();
    grid_dep_launch();
    if (NORM) {
        const float* xf = static_cast<const float*>(xin);
        float ss[TPC];
#pragma unroll
        for (int tt = 0; tt < TPC; ++tt) ss[tt] = 0.f;
        for (int i = threadIdx.x; i < H / 4; i += blockDim.x) {
#pragma unroll
            for (int tt = 0; tt < TPC; ++tt) {
                if (tt >= nt) break;
                const float4 v = __ldg(reinterpret_cast<const float4*>(xf + static_cast<size_t>(t0 + tt) * H) + i);
                ss[tt] += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
            }
        }
#pragma unroll
        for (int tt = 0; tt < TPC; ++tt) {
            ss[tt] = warp_sum(ss[tt]);
            if (lane == 0) red[tt][warp] = ss[tt];
        }
        __syncthreads();
        float inv[TPC];
#pragma unroll
        for (int tt = 0; tt < TPC; ++tt) {
            float tot = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) tot += red[tt][i];
            inv[tt] = 1.0f / sqrtf(tot / static_cast<float>(H) + eps);
        }
        for (int i = threadIdx.x; i < H / 4; i += blockDim.x) {
#pragma unroll
            for (int tt = 0; tt < TPC; ++tt) {
                if (tt >= nt) break;
                const float4 v = __ldg(reinterpret_cast<const float4*>(xf + static_cast<size_t>(t0 + tt) * H) + i);
                const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x * inv[tt], v.y * inv[tt]);
                const __nv_bfloat162 hi = __floats2bfloat162_rn(v.z * inv[tt], v.w * inv[tt]);
                float* x4 = xs + tt * H + 4 * i;
                x4[0] = __low2float(lo);
                x4[1] = __high2float(lo);
                x4[2] = __low2float(hi);
                x4[3] = __high2float(hi);
                if (rank == 0) {
                    __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(xhat_out + static_cast<size_t>(t0 + tt) * H);
                    o[2 * i] = lo;
                    o[2 * i + 1] = hi;
                }
            }
        }
    } else {
        for (int i = threadIdx.x; i < H / 8; i += blockDim.x) {
#pragma unroll
            for (int tt = 0; tt < TPC; ++tt) {
                if (tt >= nt) break;
                const uint4 u = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(xin) +
                                                                     static_cast<size_t>(t0 + tt) * H) + i);
                const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    xs[tt * H + 8 * i + 2 * j] = __uint_as_float(q[j] << 16);
                    xs[tt * H + 8 * i + 2 * j + 1] = __uint_as_float(q[j] & 0xffff0000u);
                }
            }
        }
    }
    __syncthreads();
    for (int e = e0 + warp; e < e1; e += 8) {
        const float4* wrow = reinterpret_cast<const float4*>(wr + static_cast<size_t>(e) * H);
        float acc[TPC];
#pragma unroll
        for (int tt = 0; tt < TPC; ++tt) acc[tt] = 0.f;
        if (wpre && e == e0 + warp) {
#pragma unroll
            for (int j = 0; j < RC_WPRE; ++j) {
                const int h4 = lane + 32 * j;
                if (h4 < H / 4) {
#pragma unroll
                    for (int tt = 0; tt < TPC; ++tt) {
                        const float4 b = *reinterpret_cast<const float4*>(xs + tt * H + 4 * h4);
                        acc[tt] = fmaf(wv[j].x, b.x, acc[tt]);
                        acc[tt] = fmaf(wv[j].y, b.y, acc[tt]);
                        acc[tt] = fmaf(wv[j].z, b.z, acc[tt]);
                        acc[tt] = fmaf(wv[j].w, b.w, acc[tt]);
                    }
                }
            }
        } else {
#pragma unroll 4
            for (int h4 = lane; h4 < H / 4; h4 += 32) {
                const float4 a = __ldg(wrow + h4);
#pragma unroll
                for (int tt = 0; tt < TPC; ++tt) {
                    const float4 b = *reinterpret_cast<const float4*>(xs + tt * H + 4 * h4);
                    acc[tt] = fmaf(a.x, b.x, acc[tt]);
                    acc[tt] = fmaf(a.y, b.y, acc[tt]);
                    acc[tt] = fmaf(a.z, b.z, acc[tt]);
                    acc[tt] = fmaf(a.w, b.w, acc[tt]);
                }
            }
        }
#pragma unroll
        for (int tt = 0; tt < TPC; ++tt) {
            const float sum = warp_sum(acc[tt]);
            if (lane == 0 && tt < nt)
                st_cluster_f32(&z[tt * E + e], 0,
                               bias ? sum + __ldg(bias + static_cast<size_t>(t0 + tt) * E + e) : sum);
        }
    }
    cluster_sync_all();
    if (rank == 0 && warp < nt)
        warp_topk_softmax(z + warp * E, E, k, renorm, idx + static_cast<size_t>(t0 + warp) * k,
                          w + static_cast<size_t>(t0 + warp) * k, lane);
}

// Tokens per cluster: one for small batches (the latency of one token's
// chain), four above 32 tokens, where a W_r row read once serves four tokens
// and the grid has a quarter of the CTAs.
constexpr int RC_TPC = 4;

template <bool NORM>
static ms_status route_cluster_launch_t(const void* xin, float eps, const float* wr, const float* bias, int T, int H,
                                        int E, int k, int renorm, int32_t* idx, float* w, __nv_bfloat16* xo,
                                        cudaStream_t s) {
    static PerDevice set;
    set.get([] {
        cudaFuncSetAttribute(route_cluster_kernel<NORM, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
        cudaFuncSetAttribute(route_cluster_kernel<NORM, RC_TPC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             200 * 1024);
        return 1;
    });
    if (T > 32) {
        const size_t smem = sizeof(float) * static_cast<size_t>(RC_TPC) * (H + E);
        return launch_cluster(K_ROUTE_CLUSTER, route_cluster_kernel<NORM, RC_TPC>,
                              dim3(RC_CTAS, (T + RC_TPC - 1) / RC_TPC), dim3(256), smem, s, RC_CTAS, xin, wr, bias,
                              T, H, E, k, renorm, eps, idx, w, xo);
    }
    const size_t smem = sizeof(float) * static_cast<size_t>(H + E);
    return launch_cluster(K_ROUTE_CLUSTER, route_cluster_kernel<NORM, 1>, dim3(RC_CTAS, T), dim3(256), smem, s,
                          RC_CTAS, xin, wr, bias, T, H, E, k, renorm, eps, idx, w, xo);
}

ms_status route_cluster_launch(const void* xin, bool norm, float eps, const float* wr, const float* bias, int T,
                               int H, int E, int k, int renorm, int32_t* idx, float* w, void* xhat_out,
                               cudaStream_t s) {
    auto* xo = reinterpret_cast<__nv_bfloat16*>(xhat_out);
    if (norm) return route_cluster_launch_t<true>(xin, eps, wr, bias, T, H, E, k, renorm, idx, w, xo, s);
    return route_cluster_launch_t<false>(xin, eps, wr, bias, T, H, E, k, renorm, idx, w, xo, s);
}

ms_status route_launch(const void* x, const float* wr, const float* bias, int T, int H, int E,
                       int k, int renorm, int32_t* idx, float* w, cudaStream_t s) {
    const __nv_bfloat16* xb = reinterpret_cast<const __nv_bfloat16*>(x);
    if (T < 1024) return route_cluster_launch(x, false, 0.f, wr, bias, T, H, E, k, renorm, idx, w, nullptr, s);
    if (E <= RT_EXP && H % RT_K == 0) {
        dim3 grid((T + RT_TOK - 1) / RT_TOK);
        return launch(K_ROUTE_TILED, route_tiled_kernel, grid, dim3(256), 0, s, xb, wr, bias, T, H,
                      E, k, renorm, idx, w);
    }
    const size_t smem = sizeof(float) * static_cast<size_t>(H + E);
    if (smem > 48 * 1024) {
        static PerDevice set;
        set.get([] {
            cudaFuncSetAttribute(route_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
            return 1;
        });
    }
    return launch(K_ROUTE_ROWS, route_rows_kernel, dim3(T), dim3(256), smem, s, xb, wr, bias, T,
                  H, E, k, renorm, idx, w);
}

}  // namespace ms

extern "C" ms_status moe_route_topk(const void* xhat, const float* w_router,
                                    const float* logit_bias, int T, int H, int E, int k,
                                    int renormalize, int32_t* topk_idx, float* topk_w,
                                    void* stream) {
    if (!xhat || !w_router || !topk_idx || !topk_w) return MS_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return MS_ERR_INVALID_ARG;
    if (E > ms::kMaxExperts || k > 32 || H % 128 != 0 || H > 48 * 1024) return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(xhat) || !ms::aligned16(w_router)) return MS_ERR_INVALID_ARG;
    return ms::route_launch(xhat, w_router, logit_bias, T, H, E, k, renormalize, topk_idx, topk_w,
                            static_cast<cudaStream_t>(stream));
}

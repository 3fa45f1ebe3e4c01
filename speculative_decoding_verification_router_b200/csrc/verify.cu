// a6: greedy verification of one speculative step.
//
// The verifier picks its own greedy token at each of the K+1 positions,
// accepts the longest prefix of drafts that agrees with those picks and
// commits one more token of its own (jina.ai, "Modèle et entraînement";
// clawpit.io, "Speculative decoding without accuracy loss"), so every step
// commits between 1 and K+1 tokens.
//
// Kernel 1 splits every logits row into P chunks; each block streams its
// chunk with 16-byte loads and reduces (max, lowest index).  Kernel 2, one
// warp per sequence, merges the P partials per row and runs the prefix match.
#include <math.h>

#include <mutex>

#include "ms_common.cuh"

namespace ms {

constexpr int VF_THREADS = 256;
constexpr int kMaxK = 8;

__device__ __forceinline__ void vec_load(const float* p, float (&v)[4]) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
__device__ __forceinline__ void vec_load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t q[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        v[2 * i] = __uint_as_float(q[i] << 16);
        v[2 * i + 1] = __uint_as_float(q[i] & 0xffff0000u);
    }
}
__device__ __forceinline__ float scalar_load(const float* p) { return __ldg(p); }
__device__ __forceinline__ float scalar_load(const __nv_bfloat16* p) {
    return bf16_to_f32(__ldg(reinterpret_cast<const uint16_t*>(p)));
}

template <typename TL>
__global__ void __launch_bounds__(VF_THREADS) verify_partial_kernel(const TL* __restrict__ logits,
                                                                    int V, int P, int chunk,
                                                                    int vec_ok,
                                                                    float* __restrict__ pv,
                                                                    int32_t* __restrict__ pi) {
    constexpr int VEC = 16 / sizeof(TL);
    __shared__ float sv[VF_THREADS / 32];
    __shared__ int si[VF_THREADS / 32];
    grid_dep_wait();
    grid_dep_launch();
    const int r = blockIdx.x / P, p = blockIdx.x % P;
    const int begin = p * chunk;
    const int end = min(V, begin + chunk);
    const TL* row = logits + static_cast<size_t>(r) * V;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    int tail_begin = begin;
    if (vec_ok) {
        const int nvec = (end - begin) / VEC;
        for (int q = threadIdx.x; q < nvec; q += VF_THREADS) {
            float v[VEC];
            const int i0 = begin + q * VEC;
            vec_load(row + i0, v);
#pragma unroll
            for (int e = 0; e < VEC; ++e) argmax_merge(bv, bi, v[e], i0 + e);
        }
        tail_begin = begin + nvec * VEC;
    }
    for (int i = tail_begin + threadIdx.x; i < end; i += VF_THREADS)
        argmax_merge(bv, bi, scalar_load(row + i), i);
    warp_argmax(bv, bi);
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    if (lane == 0) {
        sv[warp] = bv;
        si[warp] = bi;
    }
    __syncthreads();
    if (warp == 0) {
        bv = lane < VF_THREADS / 32 ? sv[lane] : -INFINITY;
        bi = lane < VF_THREADS / 32 ? si[lane] : 0x7fffffff;
        warp_argmax(bv, bi);
        if (lane == 0) {
            pv[blockIdx.x] = bv;
            pi[blockIdx.x] = bi;
        }
    }
}

__global__ void __launch_bounds__(128) verify_final_kernel(const float* __restrict__ pv,
                                                           const int32_t* __restrict__ pi, int B,
                                                           int K, int P,
                                                           const int32_t* __restrict__ draft,
                                                           int32_t* __restrict__ argmax,
                                                           int32_t* __restrict__ committed,
                                                           int32_t* __restrict__ n_committed) {
    grid_dep_wait();
    grid_dep_launch();
    const int b = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (b >= B) return;
    int g[kMaxK + 1];
#pragma unroll
    for (int j = 0; j <= kMaxK; ++j) {
        if (j > K) break;
        const size_t base = (static_cast<size_t>(b) * (K + 1) + j) * P;
        float bv = -INFINITY;
        int bi = 0x7fffffff;
        for (int q = lane; q < P; q += 32) argmax_merge(bv, bi, pv[base + q], pi[base + q]);
        warp_argmax(bv, bi);
        g[j] = bi;
    }
    if (lane == 0) {
        int n = 0;
        while (n < K && __ldg(draft + static_cast<size_t>(b) * K + n) == g[n]) ++n;
        int32_t* am = argmax + static_cast<size_t>(b) * (K + 1);
        int32_t* cm = committed + static_cast<size_t>(b) * (K + 1);
        for (int j = 0; j <= K; ++j) {
            am[j] = g[j];
            cm[j] = j < n ? g[j] : (j == n ? g[n] : -1);
        }
        n_committed[b] = n + 1;
    }
}

// Greedy verification from the fused vocab head's argmax keys: keys is a
// [B(K+1)][ld] table of 64-bit keys (order key of a bf16 value << 32 | ~index);
// the largest key of a row gives its largest value and, among equal values,
// the lowest index.  One 1024-thread block per sequence: every thread takes a
// strided share of all K+1 rows at once (its loads all in flight together),
// then warp and block maxima.
constexpr int VK_THREADS = 1024;

__device__ __forceinline__ unsigned long long warp_max_u64(unsigned long long v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long w = __shfl_xor_sync(0xffffffffu, v, o);
        v = w > v ? w : v;
    }
    return v;
}

__global__ void __launch_bounds__(VK_THREADS) verify_keys_kernel(const unsigned long long* __restrict__ keys,
                                                                 int ld, int K, const int32_t* __restrict__ draft,
                                                                 int32_t* __restrict__ argmax,
                                                                 int32_t* __restrict__ committed,
                                                                 int32_t* __restrict__ n_committed) {
    __shared__ unsigned long long red[VK_THREADS / 32][kMaxK + 1];
    grid_dep_wait();
    grid_dep_launch();
    const int b = blockIdx.x;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long m[kMaxK + 1];
#pragma unroll
    for (int j = 0; j <= kMaxK; ++j) m[j] = 0;
#pragma unroll 4
    for (int q = threadIdx.x; q < ld; q += VK_THREADS) {
#pragma unroll
        for (int j = 0; j <= kMaxK; ++j)
            if (j <= K) {
                const unsigned long long v = __ldcg(keys + (static_cast<size_t>(b) * (K + 1) + j) * ld + q);
                m[j] = v > m[j] ? v : m[j];
            }
    }
#pragma unroll
    for (int j = 0; j <= kMaxK; ++j)
        if (j <= K) {
            const unsigned long long v = warp_max_u64(m[j]);
            if (lane == 0) red[warp][j] = v;
        }
    __syncthreads();
    if (threadIdx.x != 0) return;
    int g[kMaxK + 1];
#pragma unroll
    for (int j = 0; j <= kMaxK; ++j)
        if (j <= K) {
            unsigned long long v = 0;
            for (int w = 0; w < VK_THREADS / 32; ++w) v = red[w][j] > v ? red[w][j] : v;
            g[j] = static_cast<int>(0xFFFFFFFFu - static_cast<uint32_t>(v & 0xFFFFFFFFull));
        }
    int n = 0;
    while (n < K && __ldg(draft + static_cast<size_t>(b) * K + n) == g[n]) ++n;
    int32_t* am = argmax + static_cast<size_t>(b) * (K + 1);
    int32_t* cm = committed + static_cast<size_t>(b) * (K + 1);
    for (int j = 0; j <= K; ++j) {
        am[j] = g[j];
        cm[j] = j < n ? g[j] : (j == n ? g[n] : -1);
    }
    n_committed[b] = n + 1;
}

ms_status verify_keys_launch(const unsigned long long* keys, int ld, int B, int K, const int32_t* draft,
                             int32_t* argmax, int32_t* committed, int32_t* n_committed, cudaStream_t s) {
    if (K < 0 || K > kMaxK) return MS_ERR_UNSUPPORTED;
    return launch(K_VERIFY_KEYS, verify_keys_kernel, dim3(B), dim3(VK_THREADS), 0, s, keys, ld, K, draft, argmax,
                  committed, n_committed);
}

// Single-kernel verification: one thread-block cluster per sequence, CTA r of
// the cluster scans chunk r % P of row r / P with 16-byte loads (several in
// flight per thread), reduces (max, lowest index) in the block and stores the
// result into CTA 0's shared memory; after the cluster barrier one warp of
// CTA 0 merges the P chunks of each row and runs the prefix match.
constexpr int VC_THREADS = 512;
constexpr int VC_MAX = 16;

// Merge the elements of one 16-byte vector (index i0 for its first element),
// converting each as it is compared, so that a thread keeps only the raw
// vectors of its loads in flight in registers.
__device__ __forceinline__ void merge_vec(float& bv, int& bi, const uint4& r, int i0, const __nv_bfloat16*) {
    const uint32_t q[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        argmax_merge(bv, bi, __uint_as_float(q[j] << 16), i0 + 2 * j);
        argmax_merge(bv, bi, __uint_as_float(q[j] & 0xffff0000u), i0 + 2 * j + 1);
    }
}
__device__ __forceinline__ void merge_vec(float& bv, int& bi, const uint4& r, int i0, const float*) {
    argmax_merge(bv, bi, __uint_as_float(r.x), i0);
    argmax_merge(bv, bi, __uint_as_float(r.y), i0 + 1);
    argmax_merge(bv, bi, __uint_as_float(r.z), i0 + 2);
    argmax_merge(bv, bi, __uint_as_float(r.w), i0 + 3);
}

// UNROLL: 16-byte loads in flight per thread -- 8 for small batches (latency:
// one round trip for a 64 KB chunk), 4 for large ones, where four 512-thread
// CTAs per SM must fit for the whole grid to be resident at once (B = 32,
// K = 3: 512 CTAs), which holds the kernel to 32 registers.
template <typename TL, int UNROLL>
__global__ void __launch_bounds__(VC_THREADS, UNROLL == 4 ? 4 : 1)
    verify_cluster_kernel(const TL* __restrict__ logits, int K, int V, int P, int chunk, int vec_ok,
                          const int32_t* __restrict__ draft, int32_t* __restrict__ argmax,
                          int32_t* __restrict__ committed, int32_t* __restrict__ n_committed) {
    constexpr int VEC = 16 / sizeof(TL);
    __shared__ float cv[VC_MAX];
    __shared__ int ci[VC_MAX];
    __shared__ float sv[VC_THREADS / 32];
    __shared__ int si[VC_THREADS / 32];
    grid_dep_wait();
    grid_dep_launch();
    const uint32_t rank = cluster_rank();
    const int b = blockIdx.y;
    const int j = static_cast<int>(rank) / P, pc = static_cast<int>(rank) % P;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    float bv = -INFINITY;
    int bi = 0x7fffffff;
    if (j <= K) {
        const int begin = pc * chunk;
        const int end = min(V, begin + chunk);
        const TL* row = logits + (static_cast<size_t>(b) * (K + 1) + j) * V;
        int tail_begin = begin;
        if (vec_ok && end > begin) {
            const int nvec = (end - begin) / VEC;
            // begin is a multiple of VEC and the row starts 16-byte aligned
            const uint4* rv = reinterpret_cast<const uint4*>(row + begin);
            for (int q0 = threadIdx.x; q0 < nvec; q0 += UNROLL * VC_THREADS) {
                uint4 raw[UNROLL];
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int q = q0 + u * VC_THREADS;
                    if (q < nvec) raw[u] = __ldg(rv + q);
                }
#pragma unroll
                for (int u = 0; u < UNROLL; ++u) {
                    const int q = q0 + u * VC_THREADS;
                    if (q < nvec) merge_vec(bv, bi, raw[u], begin + q * VEC, row);
                }
            }
            tail_begin = begin + nvec * VEC;
        }
        for (int i = tail_begin + threadIdx.x; i < end; i += VC_THREADS)
            argmax_merge(bv, bi, scalar_load(row + i), i);
    }
    warp_argmax(bv, bi);
    if (lane == 0) {
        sv[warp] = bv;
        si[warp] = bi;
    }
    __syncthreads();
    if (warp == 0) {
        bv = lane < VC_THREADS / 32 ? sv[lane] : -INFINITY;
        bi = lane < VC_THREADS / 32 ? si[lane] : 0x7fffffff;
        warp_argmax(bv, bi);
        if (lane == 0) {
            st_cluster_f32(&cv[rank], 0, bv);
            st_cluster_s32(&ci[rank], 0, bi);
        }
    }
    cluster_sync_all();
    if (rank == 0 && warp == 0) {
        // lane l < (K+1)*P holds chunk l; row r = chunks [r*P, r*P + P)
        const int n = (K + 1) * P;
        const float lv = lane < n ? cv[lane] : -INFINITY;
        const int li = lane < n ? ci[lane] : 0x7fffffff;
        const int dr = lane < K ? __ldg(draft + static_cast<size_t>(b) * K + lane) : -1;
        int g[kMaxK + 1];
#pragma unroll
        for (int r = 0; r <= kMaxK; ++r) {
            float mv = (lane >= r * P && lane < r * P + P) ? lv : -INFINITY;
            int mi = (lane >= r * P && lane < r * P + P) ? li : 0x7fffffff;
            warp_argmax(mv, mi);
            g[r] = mi;
        }
        // first draft position that disagrees with the verifier's pick
        const unsigned miss = __ballot_sync(0xffffffffu, lane < K && dr != g[lane < kMaxK ? lane : 0]);
        if (lane == 0) {
            const int n_acc = miss ? (__ffs(miss) - 1) : K;
            int32_t* am = argmax + static_cast<size_t>(b) * (K + 1);
            int32_t* cm = committed + static_cast<size_t>(b) * (K + 1);
            for (int r = 0; r <= K; ++r) {
                am[r] = g[r];
                cm[r] = r <= n_acc ? g[r] : -1;
            }
            n_committed[b] = n_acc + 1;
        }
    }
}

template <typename TL, int U>
static bool allow_big_clusters() {
    return cudaFuncSetAttribute(verify_cluster_kernel<TL, U>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
           cudaSuccess;
}

static int verify_cluster_size() {
    // 16-CTA clusters when the device allows them, else the portable 8
    static PerDevice cache;
    return cache.get([] {
        int cs = 8;
        if (allow_big_clusters<__nv_bfloat16, 4>() && allow_big_clusters<__nv_bfloat16, 8>() &&
            allow_big_clusters<float, 4>() && allow_big_clusters<float, 8>()) {
            cudaLaunchConfig_t cfg = {};
            cfg.gridDim = dim3(16, 1);
            cfg.blockDim = dim3(VC_THREADS);
            cudaLaunchAttribute at[1];
            at[0].id = cudaLaunchAttributeClusterDimension;
            at[0].val.clusterDim.x = 16;
            at[0].val.clusterDim.y = 1;
            at[0].val.clusterDim.z = 1;
            cfg.attrs = at;
            cfg.numAttrs = 1;
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, verify_cluster_kernel<__nv_bfloat16, 8>, &cfg) == cudaSuccess &&
                n > 0)
                cs = 16;
        }
        cudaGetLastError();
        return cs;
    });
}

static ms_status verify_cluster_launch(const void* logits, ms_dtype dt, const int32_t* draft, int B, int K, int V,
                                       int32_t* argmax, int32_t* committed, int32_t* ncom, cudaStream_t s) {
    const int eb = dt == MS_BF16 ? 2 : 4;
    const int vec = 16 / eb;
    const int cs_max = verify_cluster_size();
    int P = cs_max / (K + 1);
    const int maxP = (V + 1023) / 1024;
    if (P > maxP) P = maxP;
    if (P < 1) P = 1;
    int chunk = (V + P - 1) / P;
    chunk = (chunk + vec - 1) / vec * vec;
    P = (V + chunk - 1) / chunk;
    const int cs = (K + 1) * P;
    const int vec_ok = (V % vec == 0) && aligned16(logits);
    // one CTA per SM at most: unroll for latency; more CTAs than SMs: for occupancy
    const bool few = static_cast<long>(cs) * B <= num_sms();
    const __nv_bfloat16* lb = reinterpret_cast<const __nv_bfloat16*>(logits);
    const float* lf = reinterpret_cast<const float*>(logits);
    if (dt == MS_BF16)
        return few ? launch_cluster(K_VERIFY_CLUSTER, verify_cluster_kernel<__nv_bfloat16, 8>, dim3(cs, B),
                                    dim3(VC_THREADS), 0, s, cs, lb, K, V, P, chunk, vec_ok, draft, argmax, committed,
                                    ncom)
                   : launch_cluster(K_VERIFY_CLUSTER, verify_cluster_kernel<__nv_bfloat16, 4>, dim3(cs, B),
                                    dim3(VC_THREADS), 0, s, cs, lb, K, V, P, chunk, vec_ok, draft, argmax, committed,
                                    ncom);
    return few ? launch_cluster(K_VERIFY_CLUSTER, verify_cluster_kernel<float, 8>, dim3(cs, B), dim3(VC_THREADS), 0,
                                s, cs, lf, K, V, P, chunk, vec_ok, draft, argmax, committed, ncom)
               : launch_cluster(K_VERIFY_CLUSTER, verify_cluster_kernel<float, 4>, dim3(cs, B), dim3(VC_THREADS), 0,
                                s, cs, lf, K, V, P, chunk, vec_ok, draft, argmax, committed, ncom);
}

struct VerifyPlan {
    int P, chunk;
};

static VerifyPlan verify_plan(int B, int K, int V, int elem_bytes) {
    const int rows = B * (K + 1);
    const int vec = 16 / elem_bytes;
    const int target = 4 * num_sms();
    int P = (target + rows - 1) / rows;
    const int maxP = (V + 1023) / 1024;
    if (P > maxP) P = maxP;
    if (P < 1) P = 1;
    int chunk = (V + P - 1) / P;
    chunk = (chunk + vec - 1) / vec * vec;
    P = (V + chunk - 1) / chunk;
    return {P, chunk};
}

size_t verify_ws_bytes(int B, int K, int V) {
    // sized for the larger (fp32: more chunks) of the two element types
    VerifyPlan p4 = verify_plan(B, K, V, 4), p2 = verify_plan(B, K, V, 2);
    const int P = p4.P > p2.P ? p4.P : p2.P;
    const size_t n = static_cast<size_t>(B) * (K + 1) * P;
    return align_up(n * sizeof(float), 256) + align_up(n * sizeof(int32_t), 256);
}

ms_status verify_launch(const void* logits, ms_dtype dt, const int32_t* draft, int B, int K, int V,
                        int32_t* argmax, int32_t* committed, int32_t* ncom, void* ws,
                        cudaStream_t s) {
    const int eb = dt == MS_BF16 ? 2 : 4;
    const VerifyPlan plan = verify_plan(B, K, V, eb);
    const int rows = B * (K + 1);
    const size_t n = static_cast<size_t>(rows) * plan.P;
    float* pv = static_cast<float*>(ws);
    int32_t* pi = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + align_up(n * sizeof(float), 256));
    const int vec_ok = (V % (16 / eb) == 0) && aligned16(logits);
    ms_status st;
    if (dt == MS_BF16)
        st = launch(K_VERIFY_PARTIAL, verify_partial_kernel<__nv_bfloat16>, dim3(rows * plan.P),
                    dim3(VF_THREADS), 0, s, reinterpret_cast<const __nv_bfloat16*>(logits), V, plan.P,
                    plan.chunk, vec_ok, pv, pi);
    else
        st = launch(K_VERIFY_PARTIAL, verify_partial_kernel<float>, dim3(rows * plan.P),
                    dim3(VF_THREADS), 0, s, reinterpret_cast<const float*>(logits), V, plan.P,
                    plan.chunk, vec_ok, pv, pi);
    if (st != MS_OK) return st;
    const int warps_per_block = 4;
    return launch(K_VERIFY_FINAL, verify_final_kernel, dim3((B + warps_per_block - 1) / warps_per_block),
                  dim3(32 * warps_per_block), 0, s, static_cast<const float*>(pv),
                  static_cast<const int32_t*>(pi), B, K, plan.P, draft, argmax, committed, ncom);
}

// ---------------------------------------------------------------- no-alloc
// Scratch for spec_verify_greedy_noalloc: the per-chunk partial maxima live in
// this file-scope device array instead of a caller workspace.  Every GPU that
// loads the library holds these 128 KB (plus alignment slack) until the
// process exits.  16,384 partial entries cover every batch of up to 16,384
// verify rows (B*(K+1)) on a 148-SM B200.
constexpr size_t kNoAllocScratchBytes = 2 * 16384 * sizeof(float) + 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Host code cannot use `g_noalloc_scratch` as a pointer: in host code the name
// stands for a host-side shadow, not the device address.  The device address is
// looked up once per device, with that device current, and cached.
static ms_status noalloc_scratch(void** out) {
    static std::mutex mu;
    static void* addr[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) {
        set_cuda_error(e);
        return MS_ERR_CUDA;
    }
    if (dev < 0 || dev >= 64) return MS_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) {
            set_cuda_error(e);
            return MS_ERR_CUDA;
        }
        addr[dev] = p;
    }
    *out = addr[dev];
    return MS_OK;
}

}  // namespace ms

// Greedy verification without a caller workspace, for callers that cannot
// allocate device memory (see include/moespec.h).
extern "C" ms_status spec_verify_greedy_noalloc(const void* logits, ms_dtype logits_dtype,
                                                const int32_t* draft, int B, int K, int V,
                                                int32_t* argmax, int32_t* committed,
                                                int32_t* n_committed, void* stream) {
    if (!logits || (K > 0 && !draft) || !argmax || !committed || !n_committed) return MS_ERR_INVALID_ARG;
    if (B <= 0 || V <= 0 || K < 0) return MS_ERR_INVALID_ARG;
    if (logits_dtype != MS_F32 && logits_dtype != MS_BF16) return MS_ERR_INVALID_ARG;
    if (K > ms::kMaxK) return MS_ERR_UNSUPPORTED;
    if (static_cast<long>(B) * (K + 1) * V > (1L << 40)) return MS_ERR_UNSUPPORTED;
    // the partial maxima of this batch must fit the static scratch
    if (ms::verify_ws_bytes(B, K, V) > ms::kNoAllocScratchBytes) return MS_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    ms_status st = ms::noalloc_scratch(&scratch);
    if (st != MS_OK) return st;
    return ms::verify_launch(logits, logits_dtype, draft, B, K, V, argmax, committed, n_committed, scratch,
                             static_cast<cudaStream_t>(stream));
}

extern "C" size_t spec_verify_workspace_size(int B, int K, int V) {
    if (B <= 0 || K < 0 || V <= 0) return 0;
    return ms::verify_ws_bytes(B, K, V);
}

extern "C" ms_status spec_verify_greedy(const void* logits, ms_dtype logits_dtype,
                                        const int32_t* draft, int B, int K, int V,
                                        int32_t* argmax, int32_t* committed,
                                        int32_t* n_committed, void* ws, size_t ws_bytes,
                                        void* stream) {
    if (!logits || (K > 0 && !draft) || !argmax || !committed || !n_committed) return MS_ERR_INVALID_ARG;
    if (B <= 0 || V <= 0 || K < 0) return MS_ERR_INVALID_ARG;
    if (logits_dtype != MS_F32 && logits_dtype != MS_BF16) return MS_ERR_INVALID_ARG;
    if (K > ms::kMaxK) return MS_ERR_UNSUPPORTED;
    if (static_cast<long>(B) * (K + 1) * V > (1L << 40)) return MS_ERR_UNSUPPORTED;
    if (!ws || ws_bytes < ms::verify_ws_bytes(B, K, V)) return MS_ERR_WORKSPACE;
    // one cluster per sequence when its K+1 rows fit a cluster; the
    // two-kernel path (partials through ws) otherwise
    if (K + 1 <= ms::verify_cluster_size())
        return ms::verify_cluster_launch(logits, logits_dtype, draft, B, K, V, argmax, committed, n_committed,
                                         static_cast<cudaStream_t>(stream));
    return ms::verify_launch(logits, logits_dtype, draft, B, K, V, argmax, committed, n_committed,
                             ws, static_cast<cudaStream_t>(stream));
}

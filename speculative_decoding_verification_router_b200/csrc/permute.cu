// a2: group the (token, slot) pairs by expert -- a stable counting sort.
//
// Rows end up ordered by (expert, token): pairs are visited in flattened
// (token, slot) order and every expert keeps the visit order.  Ranks inside a
// warp come from __match_any_sync + popc, ranks across warps and blocks from
// exclusive sums in a fixed order, so the result is bit-exact and
// deterministic with no order-dependent atomics.
#include "ms_common.cuh"

namespace ms {

constexpr int PM_THREADS = 512;
constexpr int PM_WARPS = PM_THREADS / 32;
constexpr int PM_PER_LANE = 8;
constexpr int PM_PER_WARP = 32 * PM_PER_LANE;          // 256 pairs
constexpr int PM_CHUNK = PM_WARPS * PM_PER_WARP;       // 4096 pairs per block
constexpr int PM_MAX_E = 256;

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Per-block histogram of the expert ids in this block's chunk.
__global__ void __launch_bounds__(PM_THREADS) permute_count_kernel(const int32_t* __restrict__ idx,
                                                                   int n, int E,
                                                                   int32_t* __restrict__ hist,
                                                                   int32_t* status) {
    __shared__ int32_t cnt[PM_MAX_E];
    grid_dep_wait();
    grid_dep_launch();
    for (int e = threadIdx.x; e < E; e += PM_THREADS) cnt[e] = 0;
    __syncthreads();
    const int base = blockIdx.x * PM_CHUNK;
    for (int q = threadIdx.x; q < PM_CHUNK; q += PM_THREADS) {
        const int i = base + q;
        if (i >= n) break;
        const int e = __ldg(idx + i);
        if (e < 0 || e >= E) {
            report_status(status, MS_ERR_DEVICE_INDEX);
            continue;
        }
        atomicAdd(&cnt[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += PM_THREADS)
        hist[static_cast<size_t>(blockIdx.x) * E + e] = cnt[e];
}

// Ranks of one block's chunk of (token, slot) pairs.  On return ex[r] is the
// expert of pair wbegin + 32 r + lane (-1 past the end or when invalid) and
// pos[r] its row in expert order.  With nblocks > 1, `hist` holds every block's
// histogram from permute_count_kernel; with one block the chunk is the whole
// input and the block computes the offsets itself.  Block `chunk` == 0 writes
// `offsets` when it is non-null.
struct SortSmem {
    int32_t wcnt[PM_WARPS][PM_MAX_E];   // per-warp counts, then per-warp bases
    int32_t base[PM_MAX_E];
    int32_t before[PM_MAX_E];
};

__device__ __forceinline__ void chunk_ranks(const int32_t* __restrict__ idx, int n, int E,
                                            const int32_t* __restrict__ hist, int nblocks, int chunk,
                                            int32_t* __restrict__ offsets, SortSmem& sm,
                                            int (&ex)[PM_PER_LANE], int (&pos)[PM_PER_LANE],
                                            int32_t* status) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int i = threadIdx.x; i < PM_WARPS * PM_MAX_E; i += PM_THREADS) (&sm.wcnt[0][0])[i] = 0;
    __syncthreads();

    const int wbegin = chunk * PM_CHUNK + warp * PM_PER_WARP;
    int rk[PM_PER_LANE];
#pragma unroll
    for (int r = 0; r < PM_PER_LANE; ++r) {
        const int i = wbegin + r * 32 + lane;
        int e = i < n ? __ldg(idx + i) : -1;
        if (i < n && (e < 0 || e >= E)) {
            report_status(status, MS_ERR_DEVICE_INDEX);
            e = -1;
        }
        const uint32_t peers = __match_any_sync(0xffffffffu, e);
        int rank = 0;
        if (e >= 0) rank = sm.wcnt[warp][e] + __popc(peers & lanemask_lt());
        __syncwarp();
        if (e >= 0 && (peers & lanemask_lt()) == 0) sm.wcnt[warp][e] += __popc(peers);
        __syncwarp();
        ex[r] = e;
        rk[r] = rank;
    }
    __syncthreads();
    // per-expert exclusive sum over warps (fixed order), block total
    for (int e = threadIdx.x; e < E; e += PM_THREADS) {
        int run = 0;
        for (int w = 0; w < PM_WARPS; ++w) {
            const int c = sm.wcnt[w][e];
            sm.wcnt[w][e] = run;
            run += c;
        }
        sm.base[e] = run;     // block total for now
    }
    __syncthreads();
    // global base of expert e for this block:
    //   sum_{e'<e} total[e'] + sum_{b'<b} hist[b'][e]
    if (nblocks > 1) {
        for (int e = warp; e < E; e += PM_WARPS) {
            int tot = 0, bef = 0;
            for (int b = lane; b < nblocks; b += 32) {
                const int h = hist[static_cast<size_t>(b) * E + e];
                tot += h;
                if (b < chunk) bef += h;
            }
            tot = __reduce_add_sync(0xffffffffu, tot);
            bef = __reduce_add_sync(0xffffffffu, bef);
            if (lane == 0) {
                sm.base[e] = tot;
                sm.before[e] = bef;
            }
        }
    } else {
        for (int e = threadIdx.x; e < E; e += PM_THREADS) sm.before[e] = 0;
    }
    __syncthreads();
    if (warp == 0) {
        // exclusive scan of the totals over experts; lane owns a run of experts
        constexpr int kPer = PM_MAX_E / 32;
        const int e0 = lane * kPer;
        int loc[kPer];
        int sum = 0;
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            loc[q] = (e0 + q < E) ? sm.base[e0 + q] : 0;
            sum += loc[q];
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
#pragma unroll
        for (int q = 0; q < kPer; ++q) {
            const int e = e0 + q;
            if (e < E) {
                if (offsets && chunk == 0) offsets[e] = run;
                sm.base[e] = run + sm.before[e];
            }
            run += loc[q];
        }
        if (offsets && chunk == 0 && lane == 31) offsets[E] = incl;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < PM_PER_LANE; ++r) {
        const int e = ex[r];
        pos[r] = e < 0 ? -1 : sm.base[e] + sm.wcnt[warp][e] + rk[r];
    }
}

// Stable scatter of one chunk per block.
__global__ void __launch_bounds__(PM_THREADS) permute_scatter_kernel(
    const int32_t* __restrict__ idx, int n, int k, int E, const int32_t* __restrict__ hist,
    int nblocks, int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token,
    int32_t* __restrict__ slot_of, int32_t* status) {
    __shared__ SortSmem sm;
    grid_dep_wait();
    grid_dep_launch();
    int ex[PM_PER_LANE], pos[PM_PER_LANE];
    chunk_ranks(idx, n, E, hist, nblocks, static_cast<int>(blockIdx.x), offsets, sm, ex, pos, status);
    const int wbegin = blockIdx.x * PM_CHUNK + (threadIdx.x >> 5) * PM_PER_WARP + (threadIdx.x & 31);
#pragma unroll
    for (int r = 0; r < PM_PER_LANE; ++r) {
        if (ex[r] < 0) continue;
        const int i = wbegin + r * 32;
        perm_token[pos[r]] = i / k;
        slot_of[i] = pos[r];
    }
}

size_t permute_ws_bytes(int T, int k, int E) {
    const long n = static_cast<long>(T) * k;
    if (n <= PM_CHUNK) return 0;
    const long nb = (n + PM_CHUNK - 1) / PM_CHUNK;
    return align_up(static_cast<size_t>(nb) * E * sizeof(int32_t) + 256, 256);
}

ms_status permute_launch(const int32_t* idx, int T, int k, int E, int32_t* offsets,
                         int32_t* perm, int32_t* slot, void* ws, int32_t* status,
                         cudaStream_t s) {
    const int n = T * k;
    const int nb = (n + PM_CHUNK - 1) / PM_CHUNK;
    int32_t* hist = nullptr;
    if (nb > 1) {
        hist = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + 256);
        if (!status) status = reinterpret_cast<int32_t*>(ws);
        ms_status st = launch(K_PERMUTE_COUNT, permute_count_kernel, dim3(nb), dim3(PM_THREADS), 0,
                              s, idx, n, E, hist, status);
        if (st != MS_OK) return st;
    }
    return launch(K_PERMUTE_SCATTER, permute_scatter_kernel, dim3(nb), dim3(PM_THREADS), 0, s, idx,
                  n, k, E, static_cast<const int32_t*>(hist), nb, offsets, perm, slot, status);
}

}  // namespace ms

extern "C" size_t moe_permute_workspace_size(int T, int k, int E) {
    if (T <= 0 || k <= 0 || E <= 0) return 0;
    return ms::permute_ws_bytes(T, k, E);
}

extern "C" ms_status moe_permute(const int32_t* topk_idx, int T, int k, int E,
                                 int32_t* expert_offsets, int32_t* perm_token, int32_t* slot_of,
                                 void* ws, size_t ws_bytes, void* stream) {
    if (!topk_idx || !expert_offsets || !perm_token || !slot_of) return MS_ERR_INVALID_ARG;
    if (T <= 0 || k <= 0 || E <= 0 || k > E) return MS_ERR_INVALID_ARG;
    if (E > ms::PM_MAX_E) return MS_ERR_UNSUPPORTED;
    if (static_cast<long>(T) * k > (1L << 30)) return MS_ERR_UNSUPPORTED;
    const size_t need = ms::permute_ws_bytes(T, k, E);
    if (need > 0 && (!ws || ws_bytes < need)) return MS_ERR_WORKSPACE;
    return ms::permute_launch(topk_idx, T, k, E, expert_offsets, perm_token, slot_of, ws, nullptr,
                              static_cast<cudaStream_t>(stream));
}

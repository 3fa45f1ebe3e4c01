// The verify-sized MoE layer (at most 128 tokens) as one persistent kernel.
//
// At these batch sizes the layer streams the weights of the experts its
// tokens chose (about 160 MB for the 4 rows of one sequence's verify step,
// 450 MB for 32 sequences: the 64 routed and 2 shared experts of clawpit.io,
// "Lean architecture with a compressed encoder", top-6), so its speed is set
// by how much of the time the memory system is kept busy.  As a chain of
// launches (normalise + route, group, gather, gate/up GEMM, its split-tile
// sums, down GEMM, its sums, combine) every launch boundary drains the
// memory pipe.  Here one CTA per SM runs every phase, the phases separated
// by grid-wide barriers, and the pipeline's ring of shared-memory stages
// keeps receiving the down projection's weights while the gate/up
// projection's split tiles are summed.
//
// Phases (every CTA, in order; "barrier" = all CTAs of the grid):
//  0  routing.  RMSNorm (eps, unit gain) of the layer input, router logits
//     z = xhat W_r^T (+ bias) in fp32 over the bf16-rounded xhat, spread over
//     the CTAs (expert x token items) and written to the workspace; barrier;
//     then EVERY CTA reads all logits and takes the softmax and top-k of each
//     token (larger logit first, equal logits to the lower expert), and
//     groups the (token, slot) pairs by (expert, token), so each CTA holds
//     the whole routing without another barrier.  With more than 16 tokens
//     the normalisation is a pass of its own (barrier) and the tokens are
//     gathered into expert order for the gate/up GEMM (barrier); with at
//     most 16 every expert's gate/up GEMM takes all the tokens (the MMA's
//     narrowest N is 16 anyway) and keeps the columns of its own.
//  1  gate/up GEMM (tcgen05, TMA, the streaming schedule of ffn_core.cuh)
//     with SwiGLU in the epilogue; split tiles leave fp32 partials.  Once the
//     producer has issued its last gate/up loads it fills the freed stages
//     with the first down-projection weights.  Barrier.
//  1b the gate/up split tiles are summed (CTA order) and SwiGLU'd -> h.  Barrier.
//  2  down GEMM from h; split tiles leave partials.  Barrier.
//  3  combine: out = residual + sum_j w_j y[slot_j] + y_shared, where the y of
//     a split down-projection tile is summed here from its partials.
// The down GEMM's schedule and the contributors of every split tile (a search
// over the schedule) are built by the epilogue warps while they wait for
// their first accumulator.
// During the routing each CTA asks L2 to prefetch a slice of the shared
// experts' weights, which no routing decision can change.
//
// Every wait is bounded (the library's wait limit); a timeout records
// MS_ERR_TIMEOUT in the status word, the CTA skips the remaining work but
// still passes every grid barrier, and the in-flight copies and MMAs are
// drained before TMEM is released (as in the stand-alone GEMM kernel).
// All CTAs must be resident at once: the grid is one CTA per SM and the
// kernel's shared memory allows no second CTA on an SM.
#include "ffn_core.cuh"
#include "layer_fused.cuh"

namespace ms {

using namespace sm100;

constexpr int LF_MAXT = 128;     // tokens: the streaming schedule's limit
constexpr int LF_MAXK = 8;       // experts per token
constexpr int LF_DENSE_T = 16;   // up to this many tokens every expert's gate/up GEMM takes all of them
constexpr int LF_LOCAL_T = 24;   // up to this many tokens every CTA takes every token's top-k itself
constexpr int LF_WARPS = NTHREADS / 32;
constexpr int LF_TPI = 16;       // router item: tokens (more than 16 tokens)
constexpr int LF_RWPRE = 12;     // float4 of a router row per lane kept in registers (H <= 1536)
constexpr int LF_MAX_SPLIT = 320;   // split tiles of one GEMM: fewer than 2 * nct (the grid is at most 160 CTAs)
constexpr int LF_LOADS = 8;      // independent global loads a thread keeps in flight when staging rows

struct LfParams {
    Params g;                    // shapes and the GEMM buffers (h, y, partials, status, limits, trace)
    const float* a;              // [T][H] layer input (residual stream)
    const float* w_router;       // [E][H] fp32
    const float* bias;           // [T][E] fp32 or null
    float* out;                  // [T][H] fp32
    float eps;
    int renorm;
    int dense;                   // T <= 16
    int t_box;                   // rows of x_pad the token boxes cover: T rounded up to 16
    __nv_bfloat16* x_pad;        // [t_box][H] xhat in bf16, zero rows T..t_box-1
    __nv_bfloat16* x_perm;       // [rows_pad][H] xhat rows in expert order (T > 16)
    int rows_pad;
    float* logits;               // [T][E] router logits
    int32_t* idx_out;            // routing as the stand-alone calls would write it (for inspection)
    float* w_out;
    int32_t* off_out;
    int32_t* perm_out;
    int32_t* slot_out;
    unsigned int* bar;           // grid-barrier counter, zero when the launch starts
    const uint8_t* pf_ptr[2];    // shared experts' weights prefetched into L2 during the routing
    size_t pf_bytes[2];
    size_t pf_per[2];            // bytes of each CTA's slice (a multiple of LF_PF_CHUNK)
    int early_down_prefetch;     // 1: the down weights enter the ring as soon as the gate/up loads are issued
};

struct LfMaps {
    Maps m1;   // gate/up: routed and shared weights, routed and shared token operands
    Maps m2;   // down:    routed and shared weights, h_perm and h_shared
};

// One stage of the ring serves both GEMMs: 32 KB of weights (gate + up tiles,
// or two consecutive k-blocks of the down projection) and the token boxes of
// two k-blocks (the gate/up GEMM uses the first).
template <int NMAX>
struct LfLayout {
    static constexpr int A_BYTES = 2 * TILE_BYTES;
    static constexpr int B_BYTES = 2 * NMAX * BK * 2;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int BY_WEIGHTS = WEIGHT_BUDGET / A_BYTES;
    static constexpr int BY_SMEM = SMEM_CAP / STAGE;
    static constexpr int ST = BY_WEIGHTS < BY_SMEM ? BY_WEIGHTS : BY_SMEM;
    static constexpr int RING = ST * STAGE;
    static constexpr int SMEM = RING + 1024;
    static_assert(STAGE % 1024 == 0, "stage buffers must stay 1024-byte aligned");
    static_assert(ST >= 2, "pipeline needs two stages");
};

// Timeline rows of the fused kernel (ms_set_device_trace): 0 gate/up GEMM
// (setup = TMEM allocated, producer / MMA / epilogue done), 1 down GEMM (setup
// = the barrier after the gate/up sums), 5 entry = the barrier before the
// gate/up sums, 7 routing and combine (0 entry, 3 the barrier after the
// logits, 6 logits loaded, 4 top-k and grouping done, 1 schedules built,
// 2 the barrier before the combine, 7 exit).
constexpr int LF_ROW_ROUTE = 7;

__device__ __forceinline__ size_t align_up_dev(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ------------------------------------------------------------ grid barrier
// Barrier number n (from 0) of this launch: every CTA adds one to *bar
// (zero when the launch starts) and waits until it reaches nct * (n + 1).
// The CTA barrier and the fence before the add release all of the CTA's
// global writes; the acquire load after the wait orders every later read of
// the CTA after them.  With `tma_reads`, TMA (the async proxy) reads next
// what other CTAs wrote with ordinary stores: a proxy fence after the acquire
// orders those reads too.  Bounded: false once the wait limit passes.
__device__ __noinline__ bool grid_barrier(unsigned int* bar, unsigned int target, uint64_t lim, volatile int* verdict,
                                          bool tma_reads) {
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        atomicAdd(bar, 1u);
        int ok = 1;
        const uint64_t t0 = global_ns();
        for (uint32_t i = 0;; ++i) {
            unsigned int v;
            asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(bar) : "memory");
            if (v >= target) break;
            if ((i & 63u) == 63u && global_ns() - t0 > lim) {
                ok = 0;
                break;
            }
        }
        if (tma_reads) asm volatile("fence.proxy.async.global;" ::: "memory");
        *verdict = ok;
    }
    __syncthreads();
    return *verdict != 0;
}

// ------------------------------------------------------------ shared experts' L2 prefetch
// The shared experts' weights do not depend on the routing.  Each CTA asks L2
// for its slice of them in LF_PF_STEPS portions, one at each step of the
// routing phase, so that the prefetch occupies part of the memory system
// while the routing's own latency-bound loads and barriers run, instead of
// saturating it at the start and delaying them.
constexpr int LF_PF_STEPS = 5;
constexpr size_t LF_PF_CHUNK = 16384;

__device__ __noinline__ void lf_prefetch_shared(const LfParams& lp, int step) {
    if (threadIdx.x != 0) return;
    for (int t2 = 0; t2 < 2; ++t2) {
        const size_t bytes = lp.pf_bytes[t2], per = lp.pf_per[t2];
        const size_t lo = per * blockIdx.x;
        if (bytes == 0 || lo >= bytes) continue;
        const uint32_t span = static_cast<uint32_t>(bytes - lo < per ? bytes - lo : per);
        const uint32_t nchunk = (span + static_cast<uint32_t>(LF_PF_CHUNK) - 1) / static_cast<uint32_t>(LF_PF_CHUNK);
        // chunks [step * n / STEPS, (step + 1) * n / STEPS) of this slice
        const uint32_t q0 = nchunk * step / LF_PF_STEPS, q1 = nchunk * (step + 1) / LF_PF_STEPS;
        for (uint32_t q = q0; q < q1; ++q) {
            const uint32_t off = q * static_cast<uint32_t>(LF_PF_CHUNK);
            const uint32_t n = span - off < LF_PF_CHUNK ? span - off : static_cast<uint32_t>(LF_PF_CHUNK);
            asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(lp.pf_ptr[t2] + lo + off), "r"(n)
                         : "memory");
        }
    }
}

// ------------------------------------------------------------ phase 0: routing
// x [rows][H] of the tokens t0.. (as fp32 values of their bf16 rounding) in
// shared memory, either normalised here from the residual rows or widened
// from x_pad.  `write_pad`: also store the bf16 rows to x_pad.
__device__ __noinline__ void lf_norm_rows(const LfParams& lp, int t0, int nt, float* xs, float* red, bool write_pad) {
    (void)red;
    const int H = lp.g.H;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // token tt on warp tt % LF_WARPS; its row stays in registers (H <= 32 * 4 * LF_RWPRE)
#pragma unroll 1
    for (int tt = warp; tt < nt; tt += LF_WARPS) {
        const float4* row = reinterpret_cast<const float4*>(lp.a + static_cast<size_t>(t0 + tt) * H);
        float4 v[LF_RWPRE];
        float ss = 0.f;
#pragma unroll
        for (int j = 0; j < LF_RWPRE; ++j) {
            const int i = lane + 32 * j;
            v[j] = i < H / 4 ? __ldg(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int j = 0; j < LF_RWPRE; ++j) ss += v[j].x * v[j].x + v[j].y * v[j].y + v[j].z * v[j].z + v[j].w * v[j].w;
        ss = warp_sum(ss);
        const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + lp.eps);
        __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(lp.x_pad + static_cast<size_t>(t0 + tt) * H);
#pragma unroll
        for (int j = 0; j < LF_RWPRE; ++j) {
            const int i = lane + 32 * j;
            if (i >= H / 4) break;
            const __nv_bfloat162 lo = __floats2bfloat162_rn(v[j].x * inv, v[j].y * inv);
            const __nv_bfloat162 hi = __floats2bfloat162_rn(v[j].z * inv, v[j].w * inv);
            float* d = xs + tt * H + 4 * i;
            d[0] = __low2float(lo);
            d[1] = __high2float(lo);
            d[2] = __low2float(hi);
            d[3] = __high2float(hi);
            if (write_pad) {
                o[2 * i] = lo;
                o[2 * i + 1] = hi;
            }
        }
    }
}

// Widen nt rows of x_pad (written by other CTAs before a grid barrier) into xs.
__device__ __noinline__ void lf_load_rows(const LfParams& lp, int t0, int nt, float* xs) {
    const int H = lp.g.H, n8 = H / 8, total = nt * n8;
#pragma unroll 1
    for (int v0 = threadIdx.x; v0 < total; v0 += LF_LOADS * NTHREADS) {
        uint4 u8[LF_LOADS];
#pragma unroll
        for (int u = 0; u < LF_LOADS; ++u) {
            const int v = v0 + u * NTHREADS;
            if (v < total) {
                const int tt = v / n8, i = v - tt * n8;
                u8[u] = __ldcg(reinterpret_cast<const uint4*>(lp.x_pad + static_cast<size_t>(t0 + tt) * H) + i);
            }
        }
#pragma unroll
        for (int u = 0; u < LF_LOADS; ++u) {
            const int v = v0 + u * NTHREADS;
            if (v >= total) break;
            const int tt = v / n8, i = v - tt * n8;
            const uint32_t q[4] = {u8[u].x, u8[u].y, u8[u].z, u8[u].w};
            float* d = xs + tt * H + 8 * i;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                d[2 * j] = __uint_as_float(q[j] << 16);
                d[2 * j + 1] = __uint_as_float(q[j] & 0xffff0000u);
            }
        }
    }
}

// Logits of experts [e0, e0 + ne) for the nt tokens in xs: (expert, token)
// pairs are dealt to the warps (pair p -> expert p % ne, token p / ne), a
// warp keeps its current router row in registers; lanes split H and a warp
// sum finishes each dot product (a fixed order: deterministic).
// wv / cur: the warp's current router row and its expert (cur = -1: none yet;
// the dense path loads its CTA's row before the dependency wait).
__device__ __forceinline__ void lf_load_router_row(const LfParams& lp, int e, int lane, float4 (&wv)[LF_RWPRE]) {
    const int H = lp.g.H;
    const float4* wrow = reinterpret_cast<const float4*>(lp.w_router + static_cast<size_t>(e) * H);
#pragma unroll
    for (int j = 0; j < LF_RWPRE; ++j) {
        const int h4 = lane + 32 * j;
        wv[j] = h4 < H / 4 ? __ldg(wrow + h4) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

__device__ __forceinline__ void lf_router_logits(const LfParams& lp, int e0, int ne, int t0, int nt, const float* xs,
                                                 float4 (&wv)[LF_RWPRE], int& cur) {
    const int H = lp.g.H, E = lp.g.E;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#pragma unroll 1
    for (int pidx = warp; pidx < ne * nt; pidx += LF_WARPS) {
        const int e = e0 + pidx % ne, tt = pidx / ne;
        if (e != cur) {
            lf_load_router_row(lp, e, lane, wv);
            cur = e;
        }
        const float* x = xs + tt * H;
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < LF_RWPRE; ++j) {
            const int h4 = lane + 32 * j;
            if (h4 < H / 4) {
                const float4 b = *reinterpret_cast<const float4*>(x + 4 * h4);
                acc = fmaf(wv[j].x, b.x, acc);
                acc = fmaf(wv[j].y, b.y, acc);
                acc = fmaf(wv[j].z, b.z, acc);
                acc = fmaf(wv[j].w, b.w, acc);
            }
        }
        acc = warp_sum(acc);
        if (lane == 0) {
            const int t = t0 + tt;
            if (lp.bias) acc += __ldg(lp.bias + static_cast<size_t>(t) * E + e);
            lp.logits[static_cast<size_t>(t) * E + e] = acc;
        }
    }
}

// Shared-memory routing state every CTA builds from the logits.
struct LfRoute {
    float w[LF_MAXT * LF_MAXK];      // gate weight of (t, j)
    int32_t slot[LF_MAXT * LF_MAXK]; // grouped row of (t, j)
    uint8_t idx[LF_MAXT * LF_MAXK];  // expert of (t, j) (E <= 256)
    int32_t off[MAX_GROUPS + 1];     // expert e owns grouped rows [off[e], off[e+1])
    uint32_t tmask[MAX_GROUPS][LF_MAXT / 32];   // tokens of expert e (bit t)
};

// Contributors of a GEMM's split tiles (the tiles after the nct * D whole
// tiles of the streaming schedule): split tile i is summed from the partial
// slots of CTAs cf[i] .. cl[i]; cpre[i] = 16-column chunks of the split
// tiles before i (the gate/up sums' work items).
struct LfSplit {
    uint8_t cf[LF_MAX_SPLIT], cl[LF_MAX_SPLIT];
    uint16_t cpre[LF_MAX_SPLIT + 1];
    int first, n;
};

// Order-preserving 32-bit key of an fp32 value: a larger value has a larger
// key (NaN is not ordered); 0 is below every finite value's key.
__device__ __forceinline__ uint32_t lf_key(float v) {
    const uint32_t u = __float_as_uint(v);
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float lf_unkey(uint32_t key) {
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}

// Softmax and top-k of token t by one warp: lane l holds the logits of
// experts l, l + 32, ... (E <= 256).  Each of the k rounds takes the largest
// logit not yet taken -- equal logits to the lower expert -- with two warp
// reductions (the largest key, then the lowest expert holding it).  The
// softmax denominator is each lane's sum in expert order, then a warp sum:
// a fixed order.  Writes idx_out[t*k + j], w_out[t*k + j].
__device__ void lf_topk_token(const LfParams& lp, int t, int lane, LfRoute* local) {
    const int E = lp.g.E, k = lp.g.k;
    constexpr int PER = (MAX_GROUPS - 1) / 32;
    const float* z = lp.logits + static_cast<size_t>(t) * E;
    uint32_t key[PER];
    float mloc = -INFINITY;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
        const int e = lane + 32 * i;
        const float v = e < E ? __ldcg(z + e) : -INFINITY;
        key[i] = e < E ? lf_key(v) : 0u;
        mloc = fmaxf(mloc, v);
    }
    const float m = lf_unkey(__reduce_max_sync(0xffffffffu, lf_key(mloc)));
    float sl = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i)
        if (key[i] != 0u) sl += expf(lf_unkey(key[i]) - m);
    const float s = warp_sum(sl);
    float psum = 0.f, pmine = 0.f;
    int imine = 0;
#pragma unroll 1
    for (int j = 0; j < k; ++j) {
        uint32_t lk = 0u;
        int le = 0x7fffffff;
#pragma unroll
        for (int i = 0; i < PER; ++i)
            if (key[i] > lk) {   // strict: the lane's lowest expert among its equal keys
                lk = key[i];
                le = lane + 32 * i;
            }
        const uint32_t best = __reduce_max_sync(0xffffffffu, lk);
        const int win = static_cast<int>(__reduce_min_sync(0xffffffffu, lk == best ? static_cast<uint32_t>(le)
                                                                                 : 0xffffffffu));
        if ((win & 31) == lane) {
#pragma unroll
            for (int i = 0; i < PER; ++i)
                if (i == (win >> 5)) key[i] = 0u;
        }
        const float p = expf(lf_unkey(best) - m) / s;
        psum += p;
        if (lane == j) {
            pmine = p;
            imine = win;
        }
    }
    if (lane < k) {
        const float wv = lp.renorm ? pmine / psum : pmine;
        if (local) {
            local->idx[t * k + lane] = static_cast<uint8_t>(imine);
            local->w[t * k + lane] = wv;
        }
        if (!local || blockIdx.x == 0) {
            lp.idx_out[static_cast<size_t>(t) * k + lane] = imine;
            lp.w_out[static_cast<size_t>(t) * k + lane] = wv;
        }
    }
}

// The grouping by (expert, token), built by every CTA from the top-k of all
// tokens (written by the warps that took them, before a grid barrier):
// expert e's rows are its tokens in increasing order, so (t, j) goes to row
// off[e] + #{t' < t routed to e}.  perm: [T*k] scratch in shared memory.
__device__ void lf_grouping(const LfParams& lp, LfRoute& r, int32_t* perm, bool local) {
    const int T = lp.g.T, E = lp.g.E, k = lp.g.k;
    const int tid = threadIdx.x;
    const int total = T * k;
#pragma unroll 1
    for (int e = tid; e < E; e += NTHREADS) {
#pragma unroll
        for (int q = 0; q < LF_MAXT / 32; ++q) r.tmask[e][q] = 0u;
    }
    __syncthreads();
    if (local) {
        // this CTA took every token's top-k itself
#pragma unroll 1
        for (int v = tid; v < total; v += NTHREADS) {
            const int t = v / k;
            atomicOr(&r.tmask[r.idx[v]][t >> 5], 1u << (t & 31));
        }
    }
#pragma unroll 1
    for (int v0 = local ? total : tid; v0 < total; v0 += LF_LOADS * NTHREADS) {
        int32_t ix[LF_LOADS];
        float wv[LF_LOADS];
#pragma unroll
        for (int u = 0; u < LF_LOADS; ++u) {
            const int v = v0 + u * NTHREADS;
            if (v < total) {
                ix[u] = __ldcg(lp.idx_out + v);
                wv[u] = __ldcg(lp.w_out + v);
            }
        }
#pragma unroll
        for (int u = 0; u < LF_LOADS; ++u) {
            const int v = v0 + u * NTHREADS;
            if (v < total) {
                const int t = v / k;
                r.idx[v] = static_cast<uint8_t>(ix[u]);
                r.w[v] = wv[u];
                atomicOr(&r.tmask[ix[u]][t >> 5], 1u << (t & 31));
            }
        }
    }
    __syncthreads();
    // expert offsets: counts from the token masks, exclusive scan by warp 0
    if (tid < 32) {
        int run = 0;
#pragma unroll 1
        for (int e0 = 0; e0 < E; e0 += 32) {
            const int e = e0 + tid;
            int cnt = 0;
            if (e < E) {
#pragma unroll
                for (int q = 0; q < LF_MAXT / 32; ++q) cnt += __popc(r.tmask[e][q]);
            }
            int incl = cnt;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += v;
            }
            if (e < E) r.off[e] = run + incl - cnt;
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) r.off[E] = run;
    }
    __syncthreads();
#pragma unroll 1
    for (int v = tid; v < total; v += NTHREADS) {
        const int t = v / k, e = r.idx[v];
        int below = 0;
#pragma unroll
        for (int q = 0; q < LF_MAXT / 32; ++q) {
            const uint32_t m = r.tmask[e][q];
            if (q < (t >> 5)) below += __popc(m);
            else if (q == (t >> 5)) below += __popc(m & ((1u << (t & 31)) - 1u));
        }
        const int row = r.off[e] + below;
        r.slot[v] = row;
        perm[row] = t;
    }
    __syncthreads();
    if (blockIdx.x == 0) {
#pragma unroll 1
        for (int v = tid; v < total; v += NTHREADS) {
            lp.slot_out[v] = r.slot[v];
            lp.perm_out[v] = perm[v];
        }
        for (int e = tid; e <= E; e += NTHREADS) lp.off_out[e] = r.off[e];
    }
}

// The largest CTA whose split range starts at or before k-step `abs`.
__device__ __forceinline__ int lf_cta_of(const Sched& sc, int nct, int abs) {
    int lo = 0, hi = nct - 1;
#pragma unroll 1
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (sc.rb[mid] <= abs) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// Split-tile table of one GEMM, filled by `n_lanes` threads (lane =
// 0..n_lanes-1, a multiple of 32 starting at a warp boundary) that
// synchronise with `sync()`; the first warp of them scans the chunk counts.
template <int MODE, typename Sync>
__device__ void lf_split_table(const Params& p, const Sched& sc, LfSplit& tb, int lane, int n_lanes, Sync sync) {
    const int ng = sc.ngroups, nt = sc.tprefix[ng], nct = gridDim.x;
    const int first = nct * dp_tiles_per_cta(nt, nct);
    const int n = nt - first;
#pragma unroll 1
    for (int i = lane; i < n; i += n_lanes) {
        const int t = first + i;
        const int g = find_group_tile(sc, t);
        const int kt = group_ktiles<MODE>(p, g);
        const int ts = sc.prefix[g] + (t - sc.tprefix[g]) * kt;
        tb.cf[i] = static_cast<uint8_t>(lf_cta_of(sc, nct, ts));
        tb.cl[i] = static_cast<uint8_t>(lf_cta_of(sc, nct, ts + kt - 1));
        tb.cpre[i + 1] = static_cast<uint16_t>((sc.rows[g] + 15) / 16);
    }
    sync();
    if (lane < 32) {
        int run = 0;
#pragma unroll 1
        for (int i0 = 0; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            const int v = i < n ? tb.cpre[i + 1] : 0;
            int incl = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int u = __shfl_up_sync(0xffffffffu, incl, o);
                if (lane >= o) incl += u;
            }
            if (i < n) tb.cpre[i + 1] = static_cast<uint16_t>(run + incl);
            run += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (lane == 0) {
            tb.first = first;
            tb.n = n;
            tb.cpre[0] = 0;
        }
    }
}

// ------------------------------------------------------------ GEMM roles
// Ring slot q (0, 1, ... over both GEMMs) uses stage q % ST with phase (q / ST) & 1.
struct LfRing {
    int q;    // next slot whose token loads the producer issues
    int qw;   // next slot whose weight loads the producer issues (qw >= q: weights issued ahead)
};

template <int MODE, int NMAX>
__device__ __forceinline__ void lf_weight_loads(const LfMaps& mp, const Params& p, const Work& w, int kt, uint32_t a,
                                                uint32_t full, bool hint, uint64_t pol) {
    auto ld = [&](uint32_t dst, const CUtensorMap* m, int y, int z) {
        if (hint) tma_load_3d_hint(dst, m, full, 0, y, z, pol);
        else tma_load_3d(dst, m, full, 0, y, z);
    };
    const bool shared = w.g == p.E;
    if (MODE == G1_STREAM) {
        const int kt_h = p.H / BK;
        int z = w.g, fl = w.n * BM;
        const CUtensorMap* wm = &mp.m1.w_a;
        if (shared) {
            z = fl / p.I;
            fl -= z * p.I;
            wm = &mp.m1.w_s;
        }
        ld(a, wm, packed_row(fl, kt, kt_h), z);
        ld(a + TILE_BYTES, wm, packed_row(p.I + fl, kt, kt_h), z);
    } else {
        const int kt_i = p.I / BK;
        const int f0 = w.n * BM;
#pragma unroll
        for (int sb = 0; sb < 2; ++sb) {
            const int kb = kt * 2 + sb, kxb = kb * BK;
            if (shared) {
                const int z = kxb / p.I;
                ld(a + sb * TILE_BYTES, &mp.m2.w_s, packed_row(f0, (kxb - z * p.I) / BK, kt_i), z);
            } else {
                ld(a + sb * TILE_BYTES, &mp.m2.w_a, packed_row(f0, kb, kt_i), w.g);
            }
        }
    }
}

// Token boxes of one k-step; arrives on `full` with their bytes.
template <int MODE, int NMAX>
__device__ __forceinline__ void lf_token_loads(const LfMaps& mp, const LfParams& lp, const Sched& sc, const Work& w,
                                               int kt, uint32_t b, uint32_t full) {
    const Params& p = lp.g;
    const bool shared = w.g == p.E;
    constexpr int kSub = MODE == G1_STREAM ? 1 : 2;
    const Maps& m = MODE == G1_STREAM ? mp.m1 : mp.m2;
    const CUtensorMap* tm = shared ? &m.tok_s : &m.tok_r;
    // the dense gate/up GEMM reads every expert's tokens from x_pad row 0
    const int row0 = (shared || (MODE == G1_STREAM && lp.dense)) ? 0 : sc.row0[w.g];
    const int nb = (sc.rows[w.g] + TOKBOX - 1) / TOKBOX;
    mbar_expect_tx(full, kSub * nb * TOKBOX * BK * 2);
#pragma unroll
    for (int sb = 0; sb < kSub; ++sb)
        for (int j = 0; j < nb; ++j)
            tma_load_3d(b + sb * NMAX * BK * 2 + j * TOKBOX * BK * 2, tm, full, (kt * kSub + sb) * BK,
                        row0 + j * TOKBOX, 0);
}

// The producer's walk of one GEMM: weights (unless issued ahead) and tokens of
// every k-step of this CTA's work.
template <int MODE, int NMAX>
__device__ bool lf_produce(const LfMaps& mp, const LfParams& lp, const Sched& sc, uint32_t sbase, uint64_t* bar_full,
                           uint64_t* bar_empty, LfRing& r, bool hint, uint64_t pol, uint64_t lim, volatile int* abort) {
    using L = LfLayout<NMAX>;
    constexpr int ST = L::ST;
    const Params& p = lp.g;
    WorkIter<MODE> it;
    it.init(p, sc, blockIdx.x, gridDim.x);
    Work w;
    while (it.next(p, sc, w)) {
        for (int i = w.k0; i < w.k1; ++i, ++r.q) {
            const int kt = kstep_of(w, i);
            const int stage = r.q % ST;
            const uint32_t a = sbase + stage * L::STAGE, full = smem_addr(&bar_full[stage]);
            if (r.q >= r.qw) {
                if (!mbar_wait(smem_addr(&bar_empty[stage]), static_cast<uint32_t>((r.q / ST) & 1) ^ 1u, lim, abort))
                    return false;
                mbar_expect_tx_only(full, L::A_BYTES);
                lf_weight_loads<MODE, NMAX>(mp, p, w, kt, a, full, hint, pol);
                r.qw = r.q + 1;
            }
            lf_token_loads<MODE, NMAX>(mp, lp, sc, w, kt, a + L::A_BYTES, full);
        }
    }
    return true;
}

// Weights of the first ST k-steps of GEMM MODE, issued into the stages the
// previous GEMM frees (its MMAs release them in order); their token boxes
// follow in lf_produce once the tokens exist.
template <int MODE, int NMAX>
__device__ bool lf_prefetch_weights(const LfMaps& mp, const LfParams& lp, const Sched& sc, uint32_t sbase,
                                    uint64_t* bar_full, uint64_t* bar_empty, LfRing& r, bool hint, uint64_t pol,
                                    uint64_t lim, volatile int* abort) {
    using L = LfLayout<NMAX>;
    constexpr int ST = L::ST;
    const Params& p = lp.g;
    WorkIter<MODE> it;
    it.init(p, sc, blockIdx.x, gridDim.x);
    Work w;
    const int qmax = r.q + ST;
    while (r.qw < qmax && it.next(p, sc, w)) {
        for (int i = w.k0; i < w.k1 && r.qw < qmax; ++i, ++r.qw) {
            const int stage = r.qw % ST;
            const uint32_t a = sbase + stage * L::STAGE, full = smem_addr(&bar_full[stage]);
            if (!mbar_wait(smem_addr(&bar_empty[stage]), static_cast<uint32_t>((r.qw / ST) & 1) ^ 1u, lim, abort))
                return false;
            mbar_expect_tx_only(full, L::A_BYTES);
            lf_weight_loads<MODE, NMAX>(mp, p, w, kstep_of(w, i), a, full, hint, pol);
        }
    }
    return true;
}

struct LfMma {
    int q, acc;
    uint32_t acc_phase;
};

template <int MODE, int NMAX>
__device__ bool lf_mma(const LfParams& lp, const Sched& sc, uint32_t sbase, uint32_t tmem_base, uint64_t* bar_full,
                       uint64_t* bar_empty, uint64_t* bar_tfull, uint64_t* bar_tempty, LfMma& m, uint64_t lim,
                       volatile int* abort) {
    using L = LfLayout<NMAX>;
    constexpr int ST = L::ST;
    constexpr int kSub = MODE == G1_STREAM ? 1 : 2;
    const Params& p = lp.g;
    WorkIter<MODE> it;
    it.init(p, sc, blockIdx.x, gridDim.x);
    Work w;
    while (it.next(p, sc, w)) {
        if (!mbar_wait(smem_addr(&bar_tempty[m.acc]), m.acc_phase ^ 1u, lim, abort)) return false;
        tc_fence_after();
        const uint32_t n_mma = static_cast<uint32_t>((sc.rows[w.g] + 15) / 16 * 16);
        const uint32_t idesc = idesc_bf16_f32(BM, n_mma);
        const uint32_t d0 = tmem_base + m.acc * 256;
        for (int kt = w.k0; kt < w.k1; ++kt, ++m.q) {
            const int stage = m.q % ST;
            if (!mbar_wait(smem_addr(&bar_full[stage]), static_cast<uint32_t>((m.q / ST) & 1), lim, abort))
                return false;
            tc_fence_after();
            const uint32_t a0 = sbase + stage * L::STAGE;
            const uint32_t b0 = a0 + L::A_BYTES;
#pragma unroll
            for (int sb = 0; sb < kSub; ++sb) {
                const uint32_t a = a0 + sb * TILE_BYTES, b = b0 + sb * NMAX * BK * 2;
#pragma unroll
                for (int kk = 0; kk < BK / 16; ++kk) {
                    const uint32_t accum = (kt > w.k0 || sb > 0 || kk > 0) ? 1u : 0u;
                    const uint64_t bd = smem_desc_sw128(b + kk * 32);
                    mma_bf16(d0, smem_desc_sw128(a + kk * 32), bd, idesc, accum);
                    if (MODE == G1_STREAM)
                        mma_bf16(d0 + 128, smem_desc_sw128(a + TILE_BYTES + kk * 32), bd, idesc, accum);
                }
            }
            mma_commit(smem_addr(&bar_empty[stage]));
        }
        mma_commit(smem_addr(&bar_tfull[m.acc]));
        m.acc ^= 1;
        if (m.acc == 0) m.acc_phase ^= 1u;
    }
    return true;
}

// Row of h_perm that token column `col` of routed group g's gate/up tile goes
// to, or -1 when the token is not routed to expert g (dense mode: the columns
// are the tokens themselves; otherwise the group's rows in order).
__device__ __forceinline__ int lf_h_row(const LfParams& lp, const LfRoute& rt, const Sched& sc, int g, int col) {
    if (!lp.dense) return col < sc.rows[g] ? sc.row0[g] + col : -1;
    const uint32_t m = rt.tmask[g][0];
    if (col >= lp.g.T || !((m >> col) & 1u)) return -1;
    return sc.row0[g] + __popc(m & ((1u << col) - 1u));
}

// Store one finished h value (SwiGLU already applied).
__device__ __noinline__ void lf_store_hv(const LfParams& lp, const LfRoute& rt, const Sched& sc, int g, int col,
                                         int f, float h) {
    const Params& p = lp.g;
    if (g == p.E) {
        if (col < p.T) p.h_sh[static_cast<size_t>(col) * (p.S * p.I) + f] = __float2bfloat16_rn(h);
        return;
    }
    const int row = lf_h_row(lp, rt, sc, g, col);
    if (row >= 0) p.h_perm[static_cast<size_t>(row) * p.I + f] = __float2bfloat16_rn(h);
}

// One finished down-projection value.
__device__ __forceinline__ void lf_store_y(const Params& p, const Sched& sc, int g, int col, int f, float v) {
    if (col >= sc.rows[g]) return;
    if (g == p.E) p.y_sh[static_cast<size_t>(col) * p.H + f] = v;
    else reinterpret_cast<float*>(p.y_perm)[static_cast<size_t>(sc.row0[g] + col) * p.H + f] = v;
}

struct LfEpi {
    int acc;
    uint32_t acc_phase;
};

template <int MODE, int NMAX>
__device__ bool lf_epilogue(const LfParams& lp, const LfRoute& rt, const Sched& sc, uint32_t tmem_base,
                            uint64_t* bar_tfull, uint64_t* bar_tempty, LfEpi& e, uint64_t lim, volatile int* abort,
                            int* go) {
    constexpr bool kG1 = MODE == G1_STREAM;
    const Params& p = lp.g;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int q4 = warp & 3;
    const int r_in = q4 * 32 + lane;
    const int etid = threadIdx.x - 64;
    const int c = blockIdx.x;
    WorkIter<MODE> it;
    it.init(p, sc, c, gridDim.x);
    Work w;
    while (it.next(p, sc, w)) {
        if (!epi_wait(smem_addr(&bar_tfull[e.acc]), e.acc_phase, lim, abort, etid, go[e.acc])) return false;
        tc_fence_after();
        const int g = w.g;
        const int rows = sc.rows[g];
        const int f = w.n * BM + r_in;
        const int nch = (rows + 15) / 16;
        const bool whole = w.k0 == 0 && w.k1 == w.kt;
        float* my_slot = nullptr;
        if (!whole) {
            const bool first = it.sk_range_begin(c) >= w.tile_start;
            my_slot = p.partials + static_cast<size_t>(2 * c + (first ? 0 : 1)) * (BM * NMAX * (kG1 ? 2 : 1));
        }
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q4 * 32) << 16) + static_cast<uint32_t>(e.acc * 256);
        for (int ch = 0; ch < nch; ++ch) {
            float va[16], vb[16];
            tmem_ld16(tbase + ch * 16, va);
            if (kG1) tmem_ld16(tbase + 128 + ch * 16, vb);
            tmem_ld_wait();
            if (!whole) {
                if (kG1) {
                    slot_store16(my_slot + slot_off<NMAX>(0, ch, r_in), va);
                    slot_store16(my_slot + slot_off<NMAX>(1, ch, r_in), vb);
                } else {
#pragma unroll
                    for (int j = 0; j < 16; ++j) my_slot[slot_off_col(ch * 16 + j, r_in)] = va[j];
                }
                continue;
            }
            // static indices only: a run-time index would put the values in
            // local memory, which (shared memory taking L1) lives in L2
            const int ncol = min(16, rows - ch * 16);
#pragma unroll
            for (int j = 0; j < 16; ++j) {
                if (j >= ncol) break;
                if (kG1) lf_store_hv(lp, rt, sc, g, ch * 16 + j, f, silu_mul(va[j], vb[j]));
                else lf_store_y(p, sc, g, ch * 16 + j, f, va[j]);
            }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&bar_tempty[e.acc]));
        e.acc ^= 1;
        if (e.acc == 0) e.acc_phase ^= 1u;
    }
    return true;
}

// ------------------------------------------------------------ gate/up split-tile sums
// Work units are (item, row) pairs, items being the (split tile, 16-column
// chunk) pairs of the gate/up GEMM; unit u goes to thread u of the grid, so a
// batch of a few tokens finishes every split tile in one round.  A unit
// issues the loads of all the tile's contributors (both halves) before it
// adds them, in CTA order.  `NQ` = 4-column groups of the chunk that hold tokens.
template <int NMAX, int NQ>
__device__ void lf_finish1_unit(const LfParams& lp, const LfRoute& rt, const Sched& sc, const LfSplit& tb, int item,
                                int r) {
    const Params& p = lp.g;
    int lo = 0, hi = tb.n - 1;   // split tile of the item: largest i with cpre[i] <= item
#pragma unroll 1
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (tb.cpre[mid] <= item) lo = mid; else hi = mid - 1;
    }
    const int i = lo, ch = item - tb.cpre[i];
    const int c_first = tb.cf[i], c_last = tb.cl[i];
    if (c_first == c_last) return;   // one CTA did the whole tile and stored it
    const int t = tb.first + i;
    const int g = find_group_tile(sc, t);
    const int kt = group_ktiles<G1_STREAM>(p, g);
    const int n = t - sc.tprefix[g];
    const int tile_start = sc.prefix[g] + n * kt;
    constexpr int CB = 8 / NQ;   // contributors per round of loads
    float va[4 * NQ], vb[4 * NQ];
#pragma unroll
    for (int q = 0; q < 4 * NQ; ++q) va[q] = vb[q] = 0.f;
    int c2 = c_first;
#pragma unroll 1
    while (c2 <= c_last) {
        const float* src[CB];
        int nb = 0;
#pragma unroll
        for (int u = 0; u < CB; ++u) src[u] = nullptr;
#pragma unroll 1
        for (; c2 <= c_last && nb < CB; ++c2) {
            const int b2 = sc.rb[c2];
            if (sc.rb[c2 + 1] <= b2) continue;   // empty range: not a contributor
            const float* sl = p.partials + static_cast<size_t>(2 * c2 + (b2 < tile_start ? 1 : 0)) * (BM * NMAX * 2);
#pragma unroll
            for (int u = 0; u < CB; ++u)
                if (u == nb) src[u] = sl;
            ++nb;
        }
        float4 xa[CB][NQ], xb[CB][NQ];
#pragma unroll
        for (int u = 0; u < CB; ++u)
            if (src[u]) {
                const float4* pa = reinterpret_cast<const float4*>(src[u] + slot_off<NMAX>(0, ch, r));
                const float4* pb = reinterpret_cast<const float4*>(src[u] + slot_off<NMAX>(1, ch, r));
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    xa[u][q] = __ldcg(pa + q);
                    xb[u][q] = __ldcg(pb + q);
                }
            }
#pragma unroll
        for (int u = 0; u < CB; ++u)
            if (src[u]) {
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    va[4 * q] += xa[u][q].x; va[4 * q + 1] += xa[u][q].y;
                    va[4 * q + 2] += xa[u][q].z; va[4 * q + 3] += xa[u][q].w;
                    vb[4 * q] += xb[u][q].x; vb[4 * q + 1] += xb[u][q].y;
                    vb[4 * q + 2] += xb[u][q].z; vb[4 * q + 3] += xb[u][q].w;
                }
            }
    }
    const int f = n * BM + r;
    const int ncol = min(4 * NQ, sc.rows[g] - ch * 16);
#pragma unroll
    for (int q = 0; q < 4 * NQ; ++q) {
        if (q >= ncol) break;
        lf_store_hv(lp, rt, sc, g, ch * 16 + q, f, silu_mul(va[q], vb[q]));
    }
}

template <int NMAX>
__device__ void lf_finish1(const LfParams& lp, const LfRoute& rt, const Sched& sc, const LfSplit& tb) {
    const int units = tb.cpre[tb.n] * BM;
    const int nthreads = gridDim.x * NTHREADS;
#pragma unroll 1
    for (int u = blockIdx.x * NTHREADS + threadIdx.x; u < units; u += nthreads) {
        const int item = u / BM, r = u - item * BM;
        // columns of the chunk that hold tokens: 4 when every chunk has at most 4 (a batch of a
        // few tokens), else all 16
        if (lp.g.T <= 4) lf_finish1_unit<NMAX, 1>(lp, rt, sc, tb, item, r);
        else lf_finish1_unit<NMAX, 4>(lp, rt, sc, tb, item, r);
    }
}

// ------------------------------------------------------------ combine
// out[t, c..c+7] = sum_j w[t,j] y[t,j][c..] + y_shared[t, c..] + a[t, c..],
// fp32.  y of a token's expert is read from y_perm when one CTA computed its
// down-projection tile whole, else summed here from the tile's contributors'
// partial slots in CTA order (the down GEMM's split tiles need no pass of
// their own).  Source s of a token (s < k: its s-th expert, s == k: the
// shared experts) is summed into `y`, all of its loads issued at once.
template <int NMAX>
__device__ __forceinline__ void lf_source8(const LfParams& lp, const LfRoute& rt, const Sched& sc, const LfSplit& tb,
                                           int t, int s, int c8, float (&y)[8]) {
    const Params& p = lp.g;
    int g, col;
    const float* whole;
    if (s < p.k) {
        const int row = rt.slot[t * p.k + s];
        g = rt.idx[t * p.k + s];
        col = row - sc.row0[g];
        whole = reinterpret_cast<const float*>(p.y_perm) + static_cast<size_t>(row) * p.H;
    } else {
        g = p.E;
        col = t;
        whole = p.y_sh + static_cast<size_t>(t) * p.H;
    }
    const int n = c8 / BM, r0 = c8 - n * BM;
    const int i = sc.tprefix[g] + n - tb.first;
    constexpr int CB = 4;
    const float* src[CB];
    int nsrc = 0;
#pragma unroll
    for (int u = 0; u < CB; ++u) src[u] = nullptr;
    if (i < 0 || tb.cf[i] == tb.cl[i]) {
        src[0] = whole + c8;
        nsrc = 1;
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) y[q] = 0.f;
    int c2 = nsrc ? 1 : tb.cf[i];
    const int c_last = nsrc ? 0 : tb.cl[i];
    const int tile_start = sc.prefix[g] + n * group_ktiles<G2_STREAM>(p, g);
#pragma unroll 1
    do {
#pragma unroll 1
        for (; c2 <= c_last && nsrc < CB; ++c2) {
            const int b2 = sc.rb[c2];
            if (sc.rb[c2 + 1] <= b2) continue;   // empty range: not a contributor
            const float* sl = p.partials + static_cast<size_t>(2 * c2 + (b2 < tile_start ? 1 : 0)) * (BM * NMAX) +
                              slot_off_col(col, r0);
#pragma unroll
            for (int u = 0; u < CB; ++u)
                if (u == nsrc) src[u] = sl;
            ++nsrc;
        }
        float4 x0[CB], x1[CB];
#pragma unroll
        for (int u = 0; u < CB; ++u)
            if (src[u]) {
                x0[u] = __ldcg(reinterpret_cast<const float4*>(src[u]));
                x1[u] = __ldcg(reinterpret_cast<const float4*>(src[u]) + 1);
            }
#pragma unroll
        for (int u = 0; u < CB; ++u)
            if (src[u]) {
                y[0] += x0[u].x; y[1] += x0[u].y; y[2] += x0[u].z; y[3] += x0[u].w;
                y[4] += x1[u].x; y[5] += x1[u].y; y[6] += x1[u].z; y[7] += x1[u].w;
                src[u] = nullptr;
            }
        nsrc = 0;
    } while (c2 <= c_last);
}

template <int NMAX>
__device__ void lf_combine(const LfParams& lp, const LfRoute& rt, const Sched& sc, const LfSplit& tb) {
    const Params& p = lp.g;
    const int T = p.T, H = p.H, k = p.k, n8 = H / 8;
    const int nsrc = k + (p.S > 0 ? 1 : 0);
    const int nct = gridDim.x;
    const int lane = threadIdx.x & 31;
    if (nsrc <= 8 && T <= LF_DENSE_T) {
        // a few tokens: eight lanes per vector, lane s sums source s; the
        // eight are combined by a fixed butterfly of shuffles, in which w_s y_s
        // enter as lanes 0..k-1 and the shared experts as lane k
        const int gw = (threadIdx.x >> 5) * nct + static_cast<int>(blockIdx.x);   // warps dealt to CTAs first
        const int nw = nct * LF_WARPS;
        const int s = lane & 7;
#pragma unroll 1
        for (int v0 = gw * 4; v0 < T * n8; v0 += nw * 4) {
            const int v = v0 + (lane >> 3);
            const bool live = v < T * n8;
            const int t = live ? v / n8 : 0, c8 = live ? (v - (v / n8) * n8) * 8 : 0;
            float y[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            if (live && s < nsrc) {
                lf_source8<NMAX>(lp, rt, sc, tb, t, s, c8, y);
                const float wj = s < k ? rt.w[t * k + s] : 1.0f;
#pragma unroll
                for (int q = 0; q < 8; ++q) y[q] *= wj;
            }
#pragma unroll
            for (int o = 4; o > 0; o >>= 1)
#pragma unroll
                for (int q = 0; q < 8; ++q) y[q] += __shfl_xor_sync(0xffffffffu, y[q], o);
            if (live && s == 0) {
                const size_t o = static_cast<size_t>(t) * H + c8;
                const float4 a0 = __ldg(reinterpret_cast<const float4*>(lp.a + o));
                const float4 a1 = __ldg(reinterpret_cast<const float4*>(lp.a + o) + 1);
                float4* op = reinterpret_cast<float4*>(lp.out + o);
                op[0] = make_float4(y[0] + a0.x, y[1] + a0.y, y[2] + a0.z, y[3] + a0.w);
                op[1] = make_float4(y[4] + a1.x, y[5] + a1.y, y[6] + a1.z, y[7] + a1.w);
            }
        }
        return;
    }
    // more tokens: a thread per vector, its sources in order
#pragma unroll 1
    for (int v = threadIdx.x * nct + static_cast<int>(blockIdx.x); v < T * n8; v += nct * NTHREADS) {
        const int t = v / n8, c8 = (v - t * n8) * 8;
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
        for (int j = 0; j < nsrc; ++j) {
            float y[8];
            lf_source8<NMAX>(lp, rt, sc, tb, t, j, c8, y);
            const float wj = j < k ? rt.w[t * k + j] : 1.0f;
#pragma unroll
            for (int q = 0; q < 8; ++q) acc[q] = fmaf(wj, y[q], acc[q]);
        }
        const size_t o = static_cast<size_t>(t) * H + c8;
        const float4 a0 = __ldg(reinterpret_cast<const float4*>(lp.a + o));
        const float4 a1 = __ldg(reinterpret_cast<const float4*>(lp.a + o) + 1);
        float4* op = reinterpret_cast<float4*>(lp.out + o);
        op[0] = make_float4(acc[0] + a0.x, acc[1] + a0.y, acc[2] + a0.z, acc[3] + a0.w);
        op[1] = make_float4(acc[4] + a1.x, acc[5] + a1.y, acc[6] + a1.z, acc[7] + a1.w);
    }
}

// ------------------------------------------------------------ the kernel
template <int NMAX>
__global__ void __launch_bounds__(NTHREADS, 1)
    moe_layer_fused_kernel(const __grid_constant__ LfMaps mp, const __grid_constant__ LfParams lp) {
    using L = LfLayout<NMAX>;
    constexpr int ST = L::ST;
    const Params& p = lp.g;
    extern __shared__ uint8_t dsmem[];
    uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar_full[ST], bar_empty[ST], bar_tfull[2], bar_tempty[2], bar_drain, bar_s2;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int drain_fail_sh;
    __shared__ volatile int gbar_sh;
    __shared__ int go_sh[2];
    __shared__ Sched s1, s2;
    __shared__ LfRoute rt;
    __shared__ LfSplit tb1, tb2;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int c = blockIdx.x, nct = gridDim.x;
    const uint32_t sbase = smem_addr(ring);
    const uint64_t lim = p.wait_limit_ns;
    const int T = p.T, E = p.E, H = p.H;
    unsigned int nbar = 0;
    auto gbar = [&](bool tma_reads) {
        ++nbar;
        if (!grid_barrier(lp.bar, nbar * static_cast<unsigned int>(nct), lim, &gbar_sh, tma_reads)) {
            if (threadIdx.x == 0) report_status(p.status, MS_ERR_TIMEOUT);
            abort_sh = 1;
        }
    };

    if (threadIdx.x == 0) {
        tstamp(p, LF_ROW_ROUTE, TS_ENTRY);
        tma_prefetch_map(&mp.m1.w_a);
        tma_prefetch_map(&mp.m1.w_s);
        tma_prefetch_map(&mp.m1.tok_r);
        tma_prefetch_map(&mp.m1.tok_s);
        tma_prefetch_map(&mp.m2.w_a);
        tma_prefetch_map(&mp.m2.w_s);
        tma_prefetch_map(&mp.m2.tok_r);
        tma_prefetch_map(&mp.m2.tok_s);
        for (int i = 0; i < ST; ++i) {
            mbar_init(smem_addr(&bar_full[i]), 1);
            mbar_init(smem_addr(&bar_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_addr(&bar_tfull[i]), 1);
            mbar_init(smem_addr(&bar_tempty[i]), 4);
        }
        mbar_init(smem_addr(&bar_drain), 1);
        mbar_init(smem_addr(&bar_s2), 1);   // the down GEMM's schedule is built
        abort_sh = 0;
        drain_fail_sh = 0;
        fence_mbar_init();
    }
    // The router weights are read-only inputs: with at most 16 tokens CTA c's
    // router row (expert c) is loaded now, before the dependency wait.
    float4 wv[LF_RWPRE];
    int wcur = -1;
    if (lp.dense && c < E) {
        lf_load_router_row(lp, c, lane, wv);
        wcur = c;
    }
    lf_prefetch_shared(lp, 0);
    // The layer input comes from the previous kernel on the stream.
    grid_dep_wait();

    // ---------------------------------------------------- phase 0: routing
    float* xs = reinterpret_cast<float*>(ring);   // the ring is idle until the gate/up GEMM
    if (lp.dense) {
        // CTA c: the logits of experts c, c + nct, ... for every token; the
        // last CTA writes x_pad (and its zero rows) for the gate/up GEMM
        const bool writer = c == nct - 1;
        if (c < E || writer) {
            lf_norm_rows(lp, 0, T, xs, xs + T * H, writer);
            if (threadIdx.x == 0) tstamp(p, 6, 0);
            if (writer) {
                for (int v = threadIdx.x; v < (lp.t_box - T) * (H / 8); v += NTHREADS)
                    reinterpret_cast<uint4*>(lp.x_pad + static_cast<size_t>(T) * H)[v] = make_uint4(0, 0, 0, 0);
            }
            __syncthreads();
            for (int e = c; e < E; e += nct) lf_router_logits(lp, e, 1, 0, T, xs, wv, wcur);
            if (threadIdx.x == 0) tstamp(p, 6, 1);
        }
    } else {
        // normalisation: token t on warp t of the grid's warps
        const float* unused = nullptr;
        (void)unused;
        for (int t = c * LF_WARPS + warp; t < T; t += nct * LF_WARPS) {
            const float4* row = reinterpret_cast<const float4*>(lp.a + static_cast<size_t>(t) * H);
            float ss = 0.f;
            for (int i = lane; i < H / 4; i += 32) {
                const float4 v = __ldg(row + i);
                ss += v.x * v.x + v.y * v.y + v.z * v.z + v.w * v.w;
            }
            ss = warp_sum(ss);
            const float inv = 1.0f / sqrtf(ss / static_cast<float>(H) + lp.eps);
            __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(lp.x_pad + static_cast<size_t>(t) * H);
            for (int i = lane; i < H / 4; i += 32) {
                const float4 v = __ldg(row + i);
                o[2 * i] = __floats2bfloat162_rn(v.x * inv, v.y * inv);
                o[2 * i + 1] = __floats2bfloat162_rn(v.z * inv, v.w * inv);
            }
        }
        if (c == nct - 1) {
            for (int v = threadIdx.x; v < (lp.t_box - T) * (H / 8); v += NTHREADS)
                reinterpret_cast<uint4*>(lp.x_pad + static_cast<size_t>(T) * H)[v] = make_uint4(0, 0, 0, 0);
        }
        gbar(false);
        // router items: (LF_WARPS experts, LF_TPI tokens)
        const int egroups = (E + LF_WARPS - 1) / LF_WARPS, tgroups = (T + LF_TPI - 1) / LF_TPI;
        for (int item = c; item < egroups * tgroups; item += nct) {
            const int e0 = (item % egroups) * LF_WARPS, t0 = (item / egroups) * LF_TPI;
            const int ne = E - e0 < LF_WARPS ? E - e0 : LF_WARPS, nt = T - t0 < LF_TPI ? T - t0 : LF_TPI;
            lf_load_rows(lp, t0, nt, xs);
            __syncthreads();
            lf_router_logits(lp, e0, ne, t0, nt, xs, wv, wcur);
            __syncthreads();
        }
    }
    gbar(false);
    if (threadIdx.x == 0) tstamp(p, LF_ROW_ROUTE, TS_FIRST_DATA);
    lf_prefetch_shared(lp, 1);
    // Every CTA of this launch has passed its own dependency wait: the next
    // kernel on the stream may be scheduled (it waits for this one to finish).
    grid_dep_launch();
    // Top-k: with a few tokens every CTA takes all of them itself (warp w the
    // tokens w, w + 6, ...) into its shared memory; with more, token t on warp
    // t of the grid, through the workspace and one more barrier.
    const bool local = T <= LF_LOCAL_T;
    if (local) {
#pragma unroll 1
        for (int t = warp; t < T; t += LF_WARPS) lf_topk_token(lp, t, lane, &rt);
        __syncthreads();
    } else {
#pragma unroll 1
        for (int t = c * LF_WARPS + warp; t < T; t += nct * LF_WARPS) lf_topk_token(lp, t, lane, nullptr);
        gbar(true);
    }
    if (threadIdx.x == 0) tstamp(p, LF_ROW_ROUTE, 6);
    lf_prefetch_shared(lp, 2);
    {
        int32_t* perm = reinterpret_cast<int32_t*>(ring);
        lf_grouping(lp, rt, perm, local);
        if (threadIdx.x == 0) tstamp(p, LF_ROW_ROUTE, 4);
        lf_prefetch_shared(lp, 3);
        if (!lp.dense) {
            // the gate/up GEMM's token rows in expert order (rows past T*k are zero)
            const int n8 = H / 8, rows = T * p.k;
            for (int r = c * LF_WARPS + warp; r < lp.rows_pad; r += nct * LF_WARPS) {
                const int t = r < rows ? perm[r] : -1;
                const uint4* src = reinterpret_cast<const uint4*>(lp.x_pad + static_cast<size_t>(t < 0 ? 0 : t) * H);
                uint4* dst = reinterpret_cast<uint4*>(lp.x_perm + static_cast<size_t>(r) * H);
                for (int i = lane; i < n8; i += 32) dst[i] = t >= 0 ? __ldcg(src + i) : make_uint4(0, 0, 0, 0);
            }
        }
    }
    // The gate/up GEMM's schedule from the routing (identical in every CTA);
    // the down GEMM's is built by the epilogue warps while the gate/up GEMM runs.
    const int ngroups = E + (p.S > 0 ? 1 : 0);
    build_schedule_g<G1_STREAM, NTHREADS>(p, s1, ngroups, [&](int g, int& rows, int& row0) {
        if (g < E) {
            row0 = rt.off[g];
            const int cnt = rt.off[g + 1] - rt.off[g];
            rows = cnt > 0 ? (lp.dense ? T : cnt) : 0;
        } else {
            rows = T;
            row0 = 0;
        }
    });
    if (threadIdx.x == 0) tstamp(p, 6, 2);
    if (!lp.dense) gbar(true);   // x_perm complete before any CTA's TMA reads it
    lf_prefetch_shared(lp, 4);
    // the ring held the routing's scratch (ordinary stores); TMA writes it next
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (threadIdx.x == 0) tstamp(p, LF_ROW_ROUTE, TS_SCHEDULE);
    if (warp == 1) {
        tmem_alloc(smem_addr(&tmem_base_sh), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = tmem_base_sh;
    if (threadIdx.x == 0) tstamp(p, G1_STREAM, TS_SETUP);

    const bool hint = p.weights_evict_first != 0;
    const uint64_t wpol = hint ? l2_policy_evict_first() : 0;
    LfRing ring_st{0, 0};
    LfMma mma_st{0, 0, 0u};
    LfEpi epi_st{0, 0u};

    // ---------------------------------------------------- phase 1: gate/up GEMM
    if (!abort_sh) {
        if (warp == 0) {
            if (lane == 0) {
                bool ok = lf_produce<G1_STREAM, NMAX>(mp, lp, s1, sbase, bar_full, bar_empty, ring_st, hint, wpol,
                                                      lim, &abort_sh);
                if (ok && lp.early_down_prefetch) {
                    ok = mbar_wait(smem_addr(&bar_s2), 0, lim, &abort_sh) &&
                         lf_prefetch_weights<G2_STREAM, NMAX>(mp, lp, s2, sbase, bar_full, bar_empty, ring_st, hint,
                                                              wpol, lim, &abort_sh);
                }
                if (!ok) {
                    report_status(p.status, MS_ERR_TIMEOUT);
                    abort_sh = 1;
                }
                tstamp(p, G1_STREAM, TS_PRODUCER_DONE);
            }
            __syncwarp();
        } else if (warp == 1) {
            if (lane == 0) {
                if (!lf_mma<G1_STREAM, NMAX>(lp, s1, sbase, tmem_base, bar_full, bar_empty, bar_tfull, bar_tempty,
                                             mma_st, lim, &abort_sh)) {
                    report_status(p.status, MS_ERR_TIMEOUT);
                    abort_sh = 1;
                }
                tstamp(p, G1_STREAM, TS_LAST_MMA);
            }
            __syncwarp();
        } else {
            // Before its first accumulator is ready the epilogue tabulates the
            // contributors of both GEMMs' split tiles (the gate/up sums and the
            // combine read them).
            const int et = threadIdx.x - 64;
            auto esync = [] { asm volatile("bar.sync 1, 128;" ::: "memory"); };
            build_schedule_g<G2_STREAM, 128>(p, s2, ngroups, [&](int g, int& rows, int& row0) {
                if (g < E) {
                    row0 = rt.off[g];
                    rows = rt.off[g + 1] - rt.off[g];
                } else {
                    rows = T;
                    row0 = 0;
                }
            }, et, esync);
            if (et == 0) {
                tstamp(p, 6, 3);
                mbar_arrive(smem_addr(&bar_s2));   // the producer may read s2 now
            }
            lf_split_table<G1_STREAM>(p, s1, tb1, et, 128, esync);
            lf_split_table<G2_STREAM>(p, s2, tb2, et, 128, esync);
            if (!lf_epilogue<G1_STREAM, NMAX>(lp, rt, s1, tmem_base, bar_tfull, bar_tempty, epi_st, lim, &abort_sh,
                                              go_sh)) {
                if (threadIdx.x == 64) report_status(p.status, MS_ERR_TIMEOUT);
                abort_sh = 1;
            }
            if (threadIdx.x == 64) tstamp(p, G1_STREAM, TS_EPI_DONE);
        }
    }
    gbar(false);
    if (threadIdx.x == 0) tstamp(p, 5, TS_ENTRY);
    if (!abort_sh) lf_finish1<NMAX>(lp, rt, s1, tb1);
    if (threadIdx.x == 5 * 32) tstamp(p, 5, TS_EXIT);
    if (threadIdx.x == 0) tstamp(p, 5, TS_SCHEDULE);
    if (threadIdx.x == 64) tstamp(p, 5, TS_SETUP);
    // With its own sums done (their loads are latency-bound and must not queue
    // behind a weight stream), the producer fills the ring with the first
    // down-projection weights while the other CTAs finish theirs.
    if (threadIdx.x == 0 && !abort_sh && !lp.early_down_prefetch) {
        if (!lf_prefetch_weights<G2_STREAM, NMAX>(mp, lp, s2, sbase, bar_full, bar_empty, ring_st, hint, wpol, lim,
                                                  &abort_sh)) {
            report_status(p.status, MS_ERR_TIMEOUT);
            abort_sh = 1;
        }
    }
    if (threadIdx.x == 0) tstamp(p, 5, TS_FIRST_DATA);
    gbar(true);
    if (threadIdx.x == 0) tstamp(p, G2_STREAM, TS_SETUP);

    // ---------------------------------------------------- phase 2: down GEMM
    if (!abort_sh) {
        if (warp == 0) {
            if (lane == 0) {
                if (!lf_produce<G2_STREAM, NMAX>(mp, lp, s2, sbase, bar_full, bar_empty, ring_st, hint, wpol, lim,
                                                 &abort_sh)) {
                    report_status(p.status, MS_ERR_TIMEOUT);
                    abort_sh = 1;
                }
                tstamp(p, G2_STREAM, TS_PRODUCER_DONE);
            }
            __syncwarp();
        } else if (warp == 1) {
            if (lane == 0) {
                if (!lf_mma<G2_STREAM, NMAX>(lp, s2, sbase, tmem_base, bar_full, bar_empty, bar_tfull, bar_tempty,
                                             mma_st, lim, &abort_sh)) {
                    report_status(p.status, MS_ERR_TIMEOUT);
                    abort_sh = 1;
                }
                tstamp(p, G2_STREAM, TS_LAST_MMA);
            }
            __syncwarp();
        } else {
            if (!lf_epilogue<G2_STREAM, NMAX>(lp, rt, s2, tmem_base, bar_tfull, bar_tempty, epi_st, lim, &abort_sh,
                                              go_sh)) {
                if (threadIdx.x == 64) report_status(p.status, MS_ERR_TIMEOUT);
                abort_sh = 1;
            }
            if (threadIdx.x == 64) tstamp(p, G2_STREAM, TS_EPI_DONE);
        }
    }
    gbar(false);
    if (threadIdx.x == 0) tstamp(p, LF_ROW_ROUTE, TS_SETUP);

    // ---------------------------------------------------- phase 3: combine
    if (!abort_sh) lf_combine<NMAX>(lp, rt, s2, tb2);

    // ---------------------------------------------------- teardown
    // Every load this CTA's producer issued lands, and every MMA completes,
    // before the TMEM is released (the normal path has consumed them all; after
    // a timeout this waits, bounded, for what is still in flight).
    if (threadIdx.x == 0) {
        for (int q = ring_st.q; q < ring_st.qw; ++q) mbar_arrive(smem_addr(&bar_full[q % ST]));
        const int q_end = ring_st.qw;
        for (int s3 = 0; s3 < ST && s3 < q_end; ++s3) {
            const int q_last = s3 + ((q_end - 1 - s3) / ST) * ST;
            if (!mbar_wait(smem_addr(&bar_full[s3]), static_cast<uint32_t>(q_last / ST) & 1u, lim, nullptr))
                drain_failed(p.status, drain_fail_sh);
        }
    } else if (threadIdx.x == 32) {
        mma_commit(smem_addr(&bar_drain));
        if (!mbar_wait(smem_addr(&bar_drain), 0, lim, nullptr)) drain_failed(p.status, drain_fail_sh);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1 && !drain_fail_sh) tmem_dealloc(tmem_base, TMEM_COLS);
    if (threadIdx.x == 0) tstamp(p, LF_ROW_ROUTE, TS_EXIT);
}

// ------------------------------------------------------------ host side
template <int NMAX>
static bool lf_resident() {
    // one CTA per SM must fit, and the grid of one CTA per SM is then resident at once
    static PerDevice cache;
    return cache.get([] {
        if (cudaFuncSetAttribute(moe_layer_fused_kernel<NMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 LfLayout<NMAX>::SMEM) != cudaSuccess) {
            cudaGetLastError();
            return -1;
        }
        int n = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, moe_layer_fused_kernel<NMAX>, NTHREADS,
                                                          LfLayout<NMAX>::SMEM) != cudaSuccess) {
            cudaGetLastError();
            return -1;
        }
        return n >= 1 ? 1 : -1;
    }) > 0;
}

// Whether the fused kernel covers this layer (otherwise the chain of launches runs).
bool layer_fused_supported(int T, int H, int E, int I, int S, int k) {
    static const bool off = [] {
        const char* e = getenv("MOESPEC_UNFUSED_LAYER");
        return e && e[0] == '1';
    }();
    if (off) return false;
    // Above 16 tokens the chain of launches measured faster (B = 32: 143 vs 188 us
    // per step): the fused kernel's normalisation pass, router items, gather and
    // their barriers outweigh the launch boundaries they replace.
    // MOESPEC_FUSED_LAYER_ALL=1 runs it up to 128 tokens (for comparison).
    static const bool all = [] {
        const char* e = getenv("MOESPEC_FUSED_LAYER_ALL");
        return e && e[0] == '1';
    }();
    if (T > (all ? LF_MAXT : LF_DENSE_T)) return false;
    if (T < 1 || T > LF_MAXT || k > LF_MAXK || E > MAX_GROUPS - 1 || H % 128 != 0 || I % 128 != 0) return false;
    if (H / 4 > 32 * LF_RWPRE) return false;                              // router row in registers
    if (2 * num_sms() > LF_MAX_SPLIT) return false;                  // split-tile tables (and 8-bit CTA ids)
    const int nmax = stream_nmax(T);
    const size_t ring = nmax == 16 ? LfLayout<16>::RING : nmax == 32 ? LfLayout<32>::RING
                      : nmax == 64 ? LfLayout<64>::RING : LfLayout<128>::RING;
    const int dense = T <= LF_DENSE_T;
    const size_t xs = static_cast<size_t>(dense ? T : LF_TPI) * H * 4 + LF_MAXT * 4;
    const size_t route = align_up(static_cast<size_t>(T) * (E + 1) * 4, 16) + static_cast<size_t>(T) * k * 4;
    if (xs > ring || route > ring) return false;
    switch (nmax) {
        case 16: return lf_resident<16>();
        case 32: return lf_resident<32>();
        case 64: return lf_resident<64>();
        default: return lf_resident<128>();
    }
}

template <int NMAX>
static ms_status lf_launch_n(const LfMaps& mp, const LfParams& lp, cudaStream_t s) {
    return launch(K_LAYER_FUSED, moe_layer_fused_kernel<NMAX>, dim3(lp.g.nct), dim3(NTHREADS), LfLayout<NMAX>::SMEM,
                  s, mp, lp);
}

ms_status layer_fused_launch(const float* a, const float* wr, const float* bias, const void* wgu, const void* wd,
                             const void* wsgu, const void* wsd, int T, int H, int E, int I, int S, int k, int renorm,
                             float eps, float* out, const LfBuffers& b, cudaStream_t s) {
    const int nmax = stream_nmax(T);
    const bool dense = T <= LF_DENSE_T;
    LfParams lp{};
    Params& p = lp.g;
    p.T = T; p.H = H; p.E = E; p.I = I; p.S = S; p.k = k; p.V = 0;
    p.bn = 128;
    p.offsets = b.off;   // non-null: group E is the shared experts' group
    p.h_perm = b.h_perm;
    p.h_sh = b.h_sh;
    p.y_perm = b.y_perm;
    p.y_bf16 = 0;
    p.y_sh = b.y_sh;
    p.partials = b.partials;
    p.nct = num_sms();
    p.weights_evict_first = evict_first_allowed();
    p.status = b.status;
    p.wait_limit_ns = wait_limit_ns();
    p.dtrace = device_trace();
    lp.a = a; lp.w_router = wr; lp.bias = bias; lp.out = out; lp.eps = eps; lp.renorm = renorm;
    lp.dense = dense ? 1 : 0;
    lp.t_box = (T + TOKBOX - 1) / TOKBOX * TOKBOX;
    lp.x_pad = b.x_pad;
    lp.x_perm = b.x_perm;
    lp.rows_pad = b.rows_pad;
    lp.logits = b.logits;
    lp.idx_out = b.idx; lp.w_out = b.w; lp.off_out = b.off; lp.perm_out = b.perm; lp.slot_out = b.slot;
    lp.bar = b.bar;
    // The down projection's first weight loads start right after the gate/up
    // loads (B = 1: 57.2 vs 59.4 us per layer with them after the gate/up sums);
    // MOESPEC_LF_LATE_DOWN=1 issues them after the sums instead (for comparison).
    static const int early = [] {
        const char* e = getenv("MOESPEC_LF_LATE_DOWN");
        return (e && e[0] == '1') ? 0 : 1;
    }();
    lp.early_down_prefetch = early;
    lp.pf_ptr[0] = static_cast<const uint8_t*>(wsgu);
    lp.pf_bytes[0] = S > 0 ? static_cast<size_t>(S) * 2 * I * H * 2 : 0;
    lp.pf_ptr[1] = static_cast<const uint8_t*>(wsd);
    lp.pf_bytes[1] = S > 0 ? static_cast<size_t>(S) * H * I * 2 : 0;
    for (int t2 = 0; t2 < 2; ++t2)
        lp.pf_per[t2] = (lp.pf_bytes[t2] / p.nct + LF_PF_CHUNK - 1) / LF_PF_CHUNK * LF_PF_CHUNK;
    const uint32_t tok_box = TOKBOX;
    LfMaps mp{};
    bool ok = make_packed_map(&mp.m1.w_a, wgu, 2 * I, H, E) &&
              make_map(&mp.m1.tok_s, b.x_pad, H, lp.t_box, 1, tok_box) &&
              (dense ? make_map(&mp.m1.tok_r, b.x_pad, H, lp.t_box, 1, tok_box)
                     : make_map(&mp.m1.tok_r, b.x_perm, H, b.rows_pad, 1, tok_box));
    ok = ok && (S > 0 ? make_packed_map(&mp.m1.w_s, wsgu, 2 * I, H, S) : make_packed_map(&mp.m1.w_s, wgu, 2 * I, H, E));
    const int hs_cols = S > 0 ? S * I : BK;
    ok = ok && make_packed_map(&mp.m2.w_a, wd, H, I, E) &&
         make_map(&mp.m2.tok_r, b.h_perm, I, b.rows_pad, 1, tok_box) &&
         make_map(&mp.m2.tok_s, b.h_sh, hs_cols, b.t_pad, 1, tok_box);
    ok = ok && (S > 0 ? make_packed_map(&mp.m2.w_s, wsd, H, I, S) : make_packed_map(&mp.m2.w_s, wd, H, I, E));
    if (!ok) return MS_ERR_CUDA;
    switch (nmax) {
        case 16: return lf_launch_n<16>(mp, lp, s);
        case 32: return lf_launch_n<32>(mp, lp, s);
        case 64: return lf_launch_n<64>(mp, lp, s);
        default: return lf_launch_n<128>(mp, lp, s);
    }
}

}  // namespace ms

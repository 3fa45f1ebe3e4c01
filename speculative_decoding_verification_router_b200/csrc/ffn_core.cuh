// Shared machinery of the streaming and tiled expert GEMMs: tile and stage
// geometry, the work schedule (data-parallel whole tiles plus a stream-K
// split region cut at equal data cost), the order in which a CTA's three
// roles walk their work, the fp32 partial-sum slots of split tiles and the
// summation that finishes them.  Used by the stand-alone GEMM kernels
// (expert_ffn.cu) and by the fused verify-layer kernel (layer_fused.cu).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdlib.h>

#include "ms_sm100.cuh"

namespace ms {

using namespace sm100;

constexpr int BM = 128;                  // MMA M
constexpr int BK = 64;                   // k per stage = one 128-byte swizzle row
constexpr int TILE_BYTES = BM * BK * 2;  // 16 KB: 128 rows x 64 bf16
constexpr int TOKBOX = 16;               // token rows per TMA box (streaming)
constexpr int NTHREADS = 192;
constexpr int MAX_GROUPS = 257;
constexpr int MAX_CTAS = 256;            // streaming grid (one CTA per SM)
constexpr int TMEM_COLS = 512;
#ifndef MS_WEIGHT_BUDGET_KB
#define MS_WEIGHT_BUDGET_KB 128
#endif
// Streaming schedule: weight bytes in flight per SM (pipeline stages x the
// weight part of a stage).  About 128 KB saturates HBM with 32 KB stages;
// more only lengthens the memory queues and delays the loads a CTA waits for.
constexpr int WEIGHT_BUDGET = MS_WEIGHT_BUDGET_KB * 1024;
// Shared memory for the stages of any schedule (the tiled one is bounded by
// this alone).
constexpr int SMEM_CAP = 200 * 1024;

enum Mode : int { G1_STREAM = 0, G2_STREAM = 1, LM_STREAM = 2, G1_TILED = 3, G2_TILED = 4, ROUTE_TILED = 5 };
// ROUTE_TILED: the router on the tensor cores -- 128-token tiles times the
// router weights split into three bf16 parts (N = 3E), softmax and top-k in
// the epilogue (one thread per token).

struct Maps {
    CUtensorMap w_a;     // routed weights  [E][rows][K] (or [1][V][H] for the vocab head)
    CUtensorMap w_s;     // shared weights  [S][rows][K]
    CUtensorMap tok_r;   // routed token operand [rows][K]
    CUtensorMap tok_s;   // shared token operand [rows][K]
};

struct Params {
    int T, H, E, I, S, k, V;
    int bn;                        // tiled GEMM2 output tile width (256 or 128)
    int mt;                        // tiled: token rows per work tile (128, or 256 for a CTA pair; 0 = 128)
    const int32_t* offsets;        // [E+1]; nullptr for the vocab head
    __nv_bfloat16* h_perm;         // [rows][I]
    __nv_bfloat16* h_sh;           // [T][S*I]
    void* y_perm;                  // [T*k][H] fp32 or bf16
    int y_bf16;
    float* y_sh;                   // [T][H]
    __nv_bfloat16* logits;         // [T][V]
    unsigned long long* amax_key;  // vocab head, fused argmax: [T][V/16] keys instead of logits (NMAX 128)
    float* partials;               // 2 partial-sum slots per CTA (streaming)
    int nct;                       // grid size of the streaming GEMM (for the finish kernel)
    int weights_evict_first;       // streaming: weight tiles are loaded with an L2 evict-first policy
    int invariant;                 // streaming: batch-invariant schedule (whole tiles, natural k order)
    const float* rbias;            // router (ROUTE_TILED): logit bias [T][E] or null
    int32_t* ridx;                 //   top-k experts [T][k]
    float* rw;                     //   their gate weights [T][k]
    int rrenorm;                   //   divide the k weights by their sum
    int32_t* status;
    uint64_t wait_limit_ns;
    uint64_t* dtrace;              // optional per-CTA timeline (see ms_set_device_trace)
};

// Timeline slots written per CTA when a device trace buffer is set.
enum TraceSlot { TS_ENTRY = 0, TS_SCHEDULE, TS_SETUP, TS_FIRST_DATA, TS_LAST_MMA, TS_EPI_DONE, TS_PRODUCER_DONE, TS_EXIT };
__device__ __forceinline__ void tstamp(const Params& p, int mode, int slot) {
    if (p.dtrace && blockIdx.x < 256) p.dtrace[(static_cast<size_t>(mode) * 256 + blockIdx.x) * 8 + slot] = global_ns();
}

template <int MODE>
struct Cfg {
    static constexpr bool kStream = MODE <= LM_STREAM;
    static constexpr bool kG1 = MODE == G1_STREAM || MODE == G1_TILED;
    // 64-wide k-blocks per pipeline stage (one schedule k-step).  GEMM1's
    // streaming stage already carries two weight tiles (gate and up rows);
    // the single-operand streaming GEMMs take two consecutive k-blocks, which
    // are one contiguous 32 KB in the packed layout: per-stage costs
    // (barrier round trips, TMA issue) are paid per 32 KB, not per 16 KB.
    static constexpr int kSub = (MODE == G2_STREAM || MODE == LM_STREAM) ? 2 : 1;
};

template <int MODE, int NMAX>
struct Layout {
    static constexpr int A_BYTES =
        Cfg<MODE>::kStream ? (Cfg<MODE>::kG1 ? 2 : Cfg<MODE>::kSub) * TILE_BYTES : TILE_BYTES;
    static constexpr int B_BYTES = Cfg<MODE>::kStream ? Cfg<MODE>::kSub * NMAX * BK * 2 : 2 * TILE_BYTES;
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int BY_WEIGHTS = Cfg<MODE>::kStream ? WEIGHT_BUDGET / A_BYTES : 8;
    static constexpr int BY_SMEM = SMEM_CAP / STAGE;
    static constexpr int STAGES_RAW = BY_WEIGHTS < BY_SMEM ? BY_WEIGHTS : BY_SMEM;
    static constexpr int STAGES = STAGES_RAW > 8 ? 8 : STAGES_RAW;
    static constexpr int SMEM = STAGES * STAGE + 1024;
    static_assert(STAGE % 1024 == 0, "stage buffers must stay 1024-byte aligned");
    static_assert(STAGES >= 2, "pipeline needs two stages");
};

// ------------------------------------------------------------ schedule
struct Sched {
    int ngroups;
    int prefix[MAX_GROUPS + 1];   // units before group g (k-steps when streaming, tiles when tiled)
    int tprefix[MAX_GROUPS + 1];  // streaming: output tiles before group g
    int rows[MAX_GROUPS];
    int row0[MAX_GROUPS];
    // streaming: fcp[g] is the cost (step_cost units) of all k-steps before
    // group g; the split region is the k-steps [sk_begin, total), and CTA c's
    // split range is the k-steps [rb[c], rb[c + 1])
    int sk_begin;
    int fcp[MAX_GROUPS + 1];
    int rb[MAX_CTAS + 1];
};

// Inclusive-to-exclusive scan of a[1..n] in place (a[0] = 0), by one warp.
__device__ __forceinline__ void warp_scan_groups(int* a, int n, int lane) {
    constexpr int kPer = (MAX_GROUPS + 31) / 32;
    int loc[kPer];
    int sum = 0;
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
        const int g = lane * kPer + q;
        loc[q] = g < n ? a[g + 1] : 0;
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
        const int g = lane * kPer + q;
        run += loc[q];
        if (g < n) a[g + 1] = run;
    }
    if (lane == 0) a[0] = 0;
}

// largest g with tprefix[g] <= t
__device__ __forceinline__ int find_group_tile(const Sched& s, int t) {
    int lo = 0, hi = s.ngroups - 1;
#pragma unroll 1
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.tprefix[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
}

template <int MODE>
__device__ __forceinline__ int group_ktiles(const Params& p, int g) {
    const bool shared = p.offsets != nullptr && g == p.E;
    constexpr int KS = BK * Cfg<MODE>::kSub;   // k per schedule step
    if (MODE == G1_STREAM || MODE == G1_TILED || MODE == LM_STREAM || MODE == ROUTE_TILED) return p.H / KS;
    return (shared ? p.S * p.I : p.I) / KS;   // GEMM2: K = intermediate width
}

template <int MODE>
__device__ __forceinline__ int group_ntiles(const Params& p, int g) {
    const bool shared = p.offsets != nullptr && g == p.E;
    if (MODE == LM_STREAM) return p.V / BM;
    if (MODE == ROUTE_TILED) return 1;
    if (MODE == G1_STREAM || MODE == G1_TILED) return (shared ? p.S * p.I : p.I) / BM;
    if (MODE == G2_STREAM) return p.H / BM;
    return p.H / p.bn;   // G2_TILED
}

// Whole tiles per CTA on the streaming schedule: every full round of tiles
// but the last, so that the split region holds the last nct .. 2 nct - 1
// tiles (all of them when NT < nct).  Each CTA's split range is then about
// one tile long, and a split tile has two or three contributors (four for
// the costliest tiles), which the finish kernel sums in one or two rounds of
// loads.
__device__ __forceinline__ int dp_tiles_per_cta(int nt, int nct) {
    const int q = nt / nct;
    return q > 0 ? q - 1 : 0;
}

// Cost of one k-step of group g on the streaming schedule, in 2 KB units of
// data the CTA moves: the weight tiles (32 KB) and the group's token boxes
// (2 KB per 16 rows and 64-wide k-block).  The token boxes come from L2, but
// a CTA's loads progress at its share of the memory system whatever their
// source, so the split ranges are cut at equal cost rather than at equal
// k-steps: a range over the shared experts' 128-token group holds fewer
// k-steps than one over a 12-token expert.
template <int MODE>
__device__ __forceinline__ int step_cost(const Sched& s, int g) {
    return 16 + Cfg<MODE>::kSub * ((s.rows[g] + TOKBOX - 1) / TOKBOX);
}

// The schedule of one launch.  `group_rows(g, rows, row0)` gives group g's
// token-operand rows and its first row; build_schedule_n reads them from the
// routing offsets in global memory, the fused layer kernel from its own
// shared-memory copy.
// NT threads build it, thread `tid` = 0..NT-1 of them (every thread of the
// CTA must call it: it contains CTA barriers).
struct CtaSync {
    __device__ void operator()() const { __syncthreads(); }
};

template <int MODE, int NT, typename GroupRows, typename Sync = CtaSync>
__device__ void build_schedule_g(const Params& p, Sched& s, int ngroups, GroupRows group_rows,
                                 int tid = static_cast<int>(threadIdx.x), Sync sync = Sync()) {
    s.ngroups = ngroups;
    const int ng = s.ngroups;
#pragma unroll 1
    for (int g = tid; g < ng; g += NT) {
        int rows, row0;
        group_rows(g, rows, row0);
        s.rows[g] = rows;
        s.row0[g] = row0;
        int units = 0, tiles = 0;
        if (rows > 0) {
            if (Cfg<MODE>::kStream) {
                tiles = group_ntiles<MODE>(p, g);
                units = tiles * group_ktiles<MODE>(p, g);
            } else {
                const int mt = p.mt ? p.mt : BM;
                units = ((rows + mt - 1) / mt) * group_ntiles<MODE>(p, g);
            }
        }
        s.prefix[g + 1] = units;   // scanned below
        s.tprefix[g + 1] = tiles;
        if (Cfg<MODE>::kStream) s.fcp[g + 1] = units * step_cost<MODE>(s, g);
    }
    sync();
    if (tid < 32) warp_scan_groups(s.prefix, ng, tid);
    else if (tid < 64) warp_scan_groups(s.tprefix, ng, tid - 32);
    else if (Cfg<MODE>::kStream && tid < 96) warp_scan_groups(s.fcp, ng, tid - 64);
    sync();
    if (Cfg<MODE>::kStream) {
        // the split region: the tiles after the nct * D whole tiles
        __shared__ int skb_cost;   // cost of the k-steps before the split region
        if (tid == 0) {
            const int nt = s.tprefix[ng];
            const int fs = p.nct * dp_tiles_per_cta(nt, p.nct);
            int skb = s.prefix[ng], cskb = s.fcp[ng];
            if (fs < nt) {
                const int g = find_group_tile(s, fs);
                skb = s.prefix[g] + (fs - s.tprefix[g]) * group_ktiles<MODE>(p, g);
                cskb = s.fcp[g] + (skb - s.prefix[g]) * step_cost<MODE>(s, g);
            }
            s.sk_begin = skb;
            skb_cost = cskb;
        }
        sync();
        // CTA c's range starts at the first k-step whose cost from the start
        // of the split region reaches c/nct of the region's cost
        const int nct = p.nct, total = s.prefix[ng];
        const long long C0 = skb_cost, C = s.fcp[ng] - C0;
        // 32-bit arithmetic when the scaled costs fit (every layer of this
        // model); 64-bit division is several times slower
        const bool narrow = static_cast<long long>(s.fcp[ng]) * nct < (1LL << 31);
#pragma unroll 1
        for (int c = tid; c <= nct; c += NT) {
            int b;
            if (c == 0 || C == 0) {
                b = s.sk_begin;
            } else if (c == nct) {
                b = total;
            } else {
                const long long x = C * c + C0 * nct;   // the target cost, times nct
                int lo = 0, hi = ng - 1;                // largest g with fcp[g] * nct <= x
#pragma unroll 1
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (static_cast<long long>(s.fcp[mid]) * nct <= x) lo = mid; else hi = mid - 1;
                }
                const long long num = x - static_cast<long long>(s.fcp[lo]) * nct;
                const long long den = static_cast<long long>(nct) * step_cost<MODE>(s, lo);
                const int d = narrow ? static_cast<int>((static_cast<uint32_t>(num) + static_cast<uint32_t>(den) - 1u) /
                                                        static_cast<uint32_t>(den))
                                     : static_cast<int>((num + den - 1) / den);
                b = max(s.prefix[lo] + d, s.sk_begin);
            }
            s.rb[c] = b;
        }
        sync();
    }
}

template <int MODE, int NT>
__device__ void build_schedule_n(const Params& p, Sched& s) {
    build_schedule_g<MODE, NT>(p, s, p.offsets == nullptr ? 1 : p.E + (p.S > 0 ? 1 : 0),
                               [&](int g, int& rows, int& row0) {
        if (p.offsets == nullptr) {
            rows = p.T;
            row0 = 0;
        } else if (g < p.E) {
            row0 = __ldg(p.offsets + g);
            rows = __ldg(p.offsets + g + 1) - row0;
            // a token reaches an expert at most once, so no group exceeds T
            // rows; the streaming schedule's token buffers hold T rows only
            if (rows < 0 || row0 < 0 || row0 + rows > p.T * p.k || (Cfg<MODE>::kStream && rows > p.T)) {
                report_status(p.status, MS_ERR_DEVICE_INDEX);
                rows = 0;
            }
        } else {
            rows = p.T;
            row0 = 0;
        }
    });
}

template <int MODE>
__device__ void build_schedule(const Params& p, Sched& s) { build_schedule_n<MODE, NTHREADS>(p, s); }

// largest g with prefix[g] <= pos (g < ngroups); groups with no work have
// prefix[g] == prefix[g+1] and are never returned for pos < total.
__device__ __forceinline__ int find_group(const Sched& s, int pos) {
    int lo = 0, hi = s.ngroups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s.prefix[mid] <= pos) lo = mid; else hi = mid - 1;
    }
    return lo;
}

struct Seg {
    int g, tile, k0, k1, kt, tile_start;   // tile: n-tile (streaming) / linear tile in group (tiled)
};

template <int MODE>
__device__ __forceinline__ Seg stream_seg(const Params& p, const Sched& s, int pos, int end) {
    Seg sg;
    sg.g = find_group(s, pos);
    sg.kt = group_ktiles<MODE>(p, sg.g);
    const int local = pos - s.prefix[sg.g];
    sg.tile = local / sg.kt;
    sg.k0 = local - sg.tile * sg.kt;
    sg.tile_start = pos - sg.k0;
    const int left = end - pos;
    sg.k1 = (sg.kt - sg.k0) < left ? sg.kt : sg.k0 + left;
    return sg;
}

// ------------------------------------------------------------ work order
// One unit of work = the k-steps [k0, k1) of one output tile, accumulated into
// one TMEM buffer.  All three roles walk the same sequence.
struct Work {
    int g, n, m0, k0, k1, kt, tile_start;
    int rot;   // whole tiles: k-steps are visited as (i + rot) % kt, i = 0..kt-1
};

// The k-step loaded/multiplied at iteration i of work item w.  Whole tiles
// start at a CTA-dependent offset so that the CTAs streaming their whole tiles
// at the same time do not all read the same k offset (same DRAM channels) at
// once; partial tiles keep their natural order.
__device__ __forceinline__ int kstep_of(const Work& w, int i) { return w.rot ? (i + w.rot) % w.kt : i; }



template <int MODE>
struct WorkIter {
    // Streaming ("data-parallel + stream-K", split part first): with NT output
    // tiles in group order and nct CTAs, CTA c owns the D = dp_tiles_per_cta
    // whole tiles [c*D, c*D + D); the k-steps of the remaining NT - nct*D
    // tiles at the end of the order (the split region) are divided into nct
    // ranges of equal cost (step_cost).  A CTA walks its split range first
    // and its whole tiles last.  Contributors to a split tile store fp32
    // partials; the finish kernel that follows the GEMM sums them and applies
    // the epilogue.
    // Tiled: tiles c, c + nct, ... (round robin).
    int c, nct, state, pos, re, dp_next, dp_end, dp_step, t, total;
    bool rotate;
    const Sched* sp;

    __device__ void init(const Params& p, const Sched& s, int c_, int nct_) {
        c = c_;
        nct = nct_;
        sp = &s;
        total = s.prefix[s.ngroups];
        if (Cfg<MODE>::kStream) {
            const int nt = s.tprefix[s.ngroups];
            const int D = dp_tiles_per_cta(nt, nct);
            dp_next = c * D;
            dp_end = dp_next + D;
            dp_step = 1;
            rotate = true;
            pos = sk_range_begin(c);
            re = sk_range_begin(c + 1);
            state = 0;
            if (p.invariant) {
                // batch-invariant: tiles c, c + nct, ... each whole, k in natural
                // order -- an output's sum does not depend on the other tokens
                dp_next = c;
                dp_end = nt;
                dp_step = nct;
                rotate = false;
                pos = re = 0;
                state = 1;
            }
        } else {
            t = c;
        }
    }
    // first k-step of CTA cc's split range
    __device__ int sk_range_begin(int cc) const { return sp->rb[cc < 0 ? 0 : (cc > nct ? nct : cc)]; }
    // The CTA whose split range holds k-step `abs` (abs in the split region):
    // the largest cc with sk_range_begin(cc) <= abs.
    __device__ int sk_cta_of(int abs) const {
        const int* rb = sp->rb;
        int lo = 0, hi = nct - 1;
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (rb[mid] <= abs) lo = mid; else hi = mid - 1;
        }
        return lo;
    }

    __device__ bool next(const Params& p, const Sched& s, Work& w) {
        if (Cfg<MODE>::kStream) {
            if (state == 0) {
                if (pos < re) {
                    const Seg sg = stream_seg<MODE>(p, s, pos, re);
                    pos += sg.k1 - sg.k0;
                    w.g = sg.g;
                    w.n = sg.tile;
                    w.m0 = 0;
                    w.k0 = sg.k0;
                    w.k1 = sg.k1;
                    w.kt = sg.kt;
                    w.tile_start = sg.tile_start;
                    w.rot = 0;
                    return true;
                }
                state = 1;
            }
            if (dp_next < dp_end) {
                const int g = find_group_tile(s, dp_next);
                w.g = g;
                w.n = dp_next - s.tprefix[g];
                w.m0 = 0;
                w.k0 = 0;
                w.kt = group_ktiles<MODE>(p, g);
                w.k1 = w.kt;
                w.tile_start = s.prefix[g] + w.n * w.kt;
                w.rot = rotate ? c % w.kt : 0;
                dp_next += dp_step;
                return true;
            }
            return false;
        } else {
            if (t >= total) return false;
            const int g = find_group(s, t);
            const int local = t - s.prefix[g];
            const int nt = group_ntiles<MODE>(p, g);
            const int m = local / nt;
            w.g = g;
            w.n = local - m * nt;
            w.m0 = m * (p.mt ? p.mt : BM);
            w.k0 = 0;
            w.kt = group_ktiles<MODE>(p, g);
            w.k1 = w.kt;
            w.tile_start = -1;
            w.rot = 0;
            t += nct;
            return true;
        }
    }
};

__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// The epilogue's wait on an accumulator: one thread waits (bounded), the
// named barrier hands its verdict to all 128 epilogue threads, so either all
// of them go on or all of them stop -- none is left waiting at a barrier.
__device__ __forceinline__ bool epi_wait(uint32_t bar, uint32_t parity, uint64_t lim, volatile int* abort,
                                         int etid, int& go) {
    if (etid == 0) go = sm100::mbar_wait(bar, parity, lim, abort) ? 1 : 0;
    epi_bar();
    return *static_cast<volatile int*>(&go) != 0;
}

// silu(g) * u with CUDA's fast exponential and division intrinsics: their
// relative error (a few units in the last fp32 place) is far below the bf16
// rounding that h receives, and the epilogue of a 128-token tile evaluates it
// 128 times per thread (the IEEE forms cost about 1 us per such tile).
// Limits: g -> -inf gives -0 (the exponential overflows to +inf, whose
// reciprocal is 0); g -> +inf gives g.
__device__ __forceinline__ float silu_mul(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// Order-preserving 16-bit key of the bf16 rounding of v: a larger value has a
// larger key, and -0 is taken as +0 (they compare equal).  NaN is not ordered.
__device__ __forceinline__ uint32_t bf16_order_key(float v) {
    uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(v));
    if (b == 0x8000u) b = 0;
    return (b & 0x8000u) ? (~b & 0xFFFFu) : (b | 0x8000u);
}

// Fused argmax of the vocab head.  In this mode the accumulator is token-major
// (TMEM lane = token, column = vocabulary row of the tile), so a thread scans
// the 16 logits of one 16-row vocabulary chunk of its own token: each is
// rounded to bf16 and mapped to (order key << 16 | 65535 - column); the
// largest such word is the chunk's largest value at its lowest index.  It is
// stored as a 64-bit key (value key << 32 | ~vocabulary index) in slot
// (t, chunk) of a [T][V/16] table, every slot written exactly once; the
// verify kernel takes the max over a row's slots: largest value, then lowest
// index.
// Fused argmax, vocabulary-major form (small T): the accumulator keeps the
// vocabulary rows in TMEM lanes, so a token's logits are spread over the 32
// lanes of each warp.  One warp max over (order key << 16 | 65535 - row) gives
// the largest value of the warp's 32 rows at its lowest row; it is stored in
// the first of the two 16-row chunk slots those rows cover, and the second
// slot gets 0, which every real key exceeds.  Called by all 32 lanes.
__device__ __forceinline__ void argmax_warp_store(unsigned long long* keys, int ld, int t, float v, int row_in_tile,
                                                  int tile, int quad, int lane) {
    uint32_t k32 = (bf16_order_key(v) << 16) | (0xFFFFu - static_cast<uint32_t>(row_in_tile));
    k32 = __reduce_max_sync(0xffffffffu, k32);
    if (lane == 0) {
        const uint32_t idx = static_cast<uint32_t>(tile) * BM + (0xFFFFu - (k32 & 0xFFFFu));
        unsigned long long* slot = keys + static_cast<size_t>(t) * ld + tile * (BM / 16) + quad * 2;
        slot[0] = (static_cast<unsigned long long>(k32 >> 16) << 32) | (0xFFFFFFFFu - idx);
        slot[1] = 0;
    }
}

__device__ __forceinline__ void argmax_chunk_store(unsigned long long* keys, int ld, int t, const float (&v)[16],
                                                   int chunk) {
    uint32_t best = 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const uint32_t k = (bf16_order_key(v[j]) << 16) | (0xFFFFu - static_cast<uint32_t>(j));
        best = k > best ? k : best;
    }
    const uint32_t idx = static_cast<uint32_t>(chunk) * 16 + (0xFFFFu - (best & 0xFFFFu));
    keys[static_cast<size_t>(t) * ld + chunk] = (static_cast<unsigned long long>(best >> 16) << 32) | (0xFFFFFFFFu - idx);
}

// Partial-sum slot of a split tile.  GEMM1 (gate and up halves):
// [half][chunk][row][16], so a thread's 16 values of one chunk are 64
// contiguous bytes and contributors write and the finisher reads with
// full-width vector accesses.  GEMM2 and the vocab head (one half):
// [column][row], so the 4 or 8 consecutive output features of one token that
// the combine kernel wants are contiguous, and a warp's stores of one column
// are 128 contiguous bytes.
template <int NMAX>
__device__ __forceinline__ size_t slot_off(int half, int ch, int r) {
    return ((static_cast<size_t>(half) * (NMAX / 16) + ch) * BM + r) * 16;
}
__device__ __forceinline__ size_t slot_off_col(int col, int r) { return static_cast<size_t>(col) * BM + r; }
__device__ __forceinline__ void slot_store16(float* dst, const float (&v)[16]) {
    float4* d = reinterpret_cast<float4*>(dst);
#pragma unroll
    for (int q = 0; q < 4; ++q) d[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}
// va += the first 4*NQ columns of chunk ch, row r, of every contributor's
// single-half slot, contributors in CTA order, 8/NQ contributors per round.
template <int NQ, typename SlotOf>
__device__ __forceinline__ void slot_sum_col(SlotOf slot_of, int c_first, int c_last, int ch, int r,
                                             float (&va)[16]) {
    constexpr int CB = 8 / NQ;
    int c2 = c_first;
    while (true) {
        const float* src[CB];
        int nb = 0;
        for (; c2 <= c_last && nb < CB; ++c2) {
            const float* sl = slot_of(c2);
            if (sl) src[nb++] = sl;
        }
        if (nb == 0) break;
        float x[CB][4 * NQ];
#pragma unroll
        for (int u = 0; u < CB; ++u)
            if (u < nb) {
#pragma unroll
                for (int j = 0; j < 4 * NQ; ++j) x[u][j] = __ldcg(src[u] + slot_off_col(ch * 16 + j, r));
            }
#pragma unroll
        for (int u = 0; u < CB; ++u)
            if (u < nb) {
#pragma unroll
                for (int j = 0; j < 4 * NQ; ++j) va[j] += x[u][j];
            }
    }
}

// va (and vb, for GEMM1's second half) += the first 4*NQ values of every
// contributor's slot of chunk ch, row r, contributors in CTA order.  The loads
// of 8/NQ contributors (both halves) are issued before any addition, so the
// usual two or three contributors cost one round trip.
template <int NMAX, int NQ, bool G1, typename SlotOf>
__device__ __forceinline__ void slot_sum(SlotOf slot_of, int c_first, int c_last, int ch, int r,
                                         float (&va)[16], float (&vb)[16]) {
    constexpr int CB = 8 / NQ;
    int c2 = c_first;
    while (true) {
        const float* src[CB];
        int nb = 0;
        for (; c2 <= c_last && nb < CB; ++c2) {
            const float* sl = slot_of(c2);
            if (sl) src[nb++] = sl;
        }
        if (nb == 0) break;
        float4 xa[CB][NQ], xb[CB][NQ];
#pragma unroll
        for (int u = 0; u < CB; ++u)
            if (u < nb) {
                const float4* pa = reinterpret_cast<const float4*>(src[u] + slot_off<NMAX>(0, ch, r));
                const float4* pb = reinterpret_cast<const float4*>(src[u] + slot_off<NMAX>(1, ch, r));
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    xa[u][q] = __ldcg(pa + q);
                    if (G1) xb[u][q] = __ldcg(pb + q);
                }
            }
#pragma unroll
        for (int u = 0; u < CB; ++u)
            if (u < nb) {
#pragma unroll
                for (int q = 0; q < NQ; ++q) {
                    va[4 * q] += xa[u][q].x; va[4 * q + 1] += xa[u][q].y;
                    va[4 * q + 2] += xa[u][q].z; va[4 * q + 3] += xa[u][q].w;
                    if (G1) {
                        vb[4 * q] += xb[u][q].x; vb[4 * q + 1] += xb[u][q].y;
                        vb[4 * q + 2] += xb[u][q].z; vb[4 * q + 3] += xb[u][q].w;
                    }
                }
            }
    }
}

// Row of the packed weight tensor (see pack.cu) that starts the 128-row x
// 64-column tile at (row r0, k-step kb) of a matrix with `kt` k-steps per row.
__device__ __forceinline__ int packed_row(int r0, int kb, int kt) { return ((r0 / BM) * kt + kb) * BM; }

// ------------------------------------------------------------ finish kernel
// Sums the parts of every tile the streaming GEMM split between CTAs (its
// contributors wrote fp32 partials and moved on) in CTA order, and applies
// that GEMM's epilogue: SwiGLU -> h for GEMM1, y for GEMM2, logits for the
// vocab head.  Running after the GEMM, it reads the partials from a quiet
// memory system instead of competing with the GEMM's weight stream.
// Work items are the (split tile, 16-column chunk) pairs whose chunk holds
// tokens (token-major argmax: all 8 chunks of 16 vocabulary rows), in tile
// order; CTA b takes items b, b + grid, ...  128 threads = the tile's rows.
// timeline row of the finish kernel that follows GEMM mode MODE
template <int MODE>
__device__ __forceinline__ void fin_stamp(const Params& p, int slot) {
    if (threadIdx.x == 0) tstamp(p, 5 + MODE, slot);
}

constexpr int FIN_THREADS = BM;

// Grid of the finish kernel: enough CTAs for every split tile of a batch of
// up to 16 tokens in one round (at most 2*nct - 1 split tiles, one chunk
// each); for larger batches two CTAs per SM (three for the vocab head),
// looping over the items: that many fit on an SM at the kernel's register
// use, so every CTA is resident at once (at B = 32 two per SM measured 143
// us per step against 148 with four and 149 with one).
template <int MODE, int NMAX>
static int finish_grid(int nct) {
    const int most = 2 * nct * (NMAX / 16);
    const int cap = (MODE == LM_STREAM ? 3 : 2) * nct;
    return most < cap ? most : cap;
}

// One item of the finish kernel: split tile t (n-th tile of group g), chunk ch.
template <int MODE, int NMAX>
__device__ __forceinline__ void finish_item(const Params& p, const Sched& sched, const WorkIter<MODE>& it, int g,
                                            int t, int ch) {
    constexpr bool kG1 = Cfg<MODE>::kG1;
    const int slot_floats = BM * NMAX * (kG1 ? 2 : 1);
    const int r = threadIdx.x;
    const int kt = group_ktiles<MODE>(p, g);
    const int n = t - sched.tprefix[g];
    const int tile_start = sched.prefix[g] + n * kt;
    const int c_first = it.sk_cta_of(tile_start), c_last = it.sk_cta_of(tile_start + kt - 1);
    if (c_first == c_last) return;   // one CTA did the whole tile and stored it
    const int rows = sched.rows[g], row0 = sched.row0[g];
    auto slot_of = [&](int c2) -> const float* {
        const int b2 = it.sk_range_begin(c2);
        if (it.sk_range_begin(c2 + 1) <= b2) return nullptr;   // empty range: not a contributor
        return p.partials + static_cast<size_t>(2 * c2 + (b2 < tile_start ? 1 : 0)) * slot_floats;
    };
    float va[16], vb[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) va[j] = vb[j] = 0.f;
    if (MODE == LM_STREAM && p.amax_key && NMAX < BM) {
        // vocabulary-major partials: thread = row r, chunk ch = 16 tokens
        const int rc = rows - ch * 16;
        if (rc <= 4) slot_sum_col<1>(slot_of, c_first, c_last, ch, r, va);
        else if (rc <= 8) slot_sum_col<2>(slot_of, c_first, c_last, ch, r, va);
        else slot_sum_col<4>(slot_of, c_first, c_last, ch, r, va);
#pragma unroll
        for (int j = 0; j < 16; ++j)
            if (ch * 16 + j < rows) argmax_warp_store(p.amax_key, p.V / 16, ch * 16 + j, va[j], r, n, r >> 5, r & 31);
        return;
    }
    if (MODE == LM_STREAM && p.amax_key) {
        // token-major partials: thread = token, chunk ch = 16 vocabulary rows
        if (r < rows) {
            slot_sum<NMAX, 4, false>(slot_of, c_first, c_last, ch, r, va, vb);
            argmax_chunk_store(p.amax_key, p.V / 16, r, va, n * (BM / 16) + ch);
        }
        return;
    }
    const int rc = rows - ch * 16;   // tokens of this chunk (only those are read)
    if (kG1) {
        if (NMAX >= 32) {
            // one load width (all 16 columns, whatever the chunk's tokens; the
            // columns past them are read and never stored): one summation
            // body keeps the kernel at ~136 registers, so the next GEMM's CTA
            // fits beside two finish CTAs on an SM and starts its weight
            // stream while the sums run
            slot_sum<NMAX, 4, true>(slot_of, c_first, c_last, ch, r, va, vb);
        } else {
            if (rc <= 4) slot_sum<NMAX, 1, true>(slot_of, c_first, c_last, ch, r, va, vb);
            else if (rc <= 8) slot_sum<NMAX, 2, true>(slot_of, c_first, c_last, ch, r, va, vb);
            else slot_sum<NMAX, 4, true>(slot_of, c_first, c_last, ch, r, va, vb);
        }
    } else {
        if (rc <= 4) slot_sum_col<1>(slot_of, c_first, c_last, ch, r, va);
        else if (rc <= 8) slot_sum_col<2>(slot_of, c_first, c_last, ch, r, va);
        else slot_sum_col<4>(slot_of, c_first, c_last, ch, r, va);
    }
    fin_stamp<MODE>(p, TS_FIRST_DATA);
    const bool shared = p.offsets != nullptr && g == p.E;
    const int f = n * BM + r;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int tok = ch * 16 + j;
        if (tok >= rows) break;
        if (MODE == G1_STREAM) {
            __nv_bfloat16* dst = shared ? p.h_sh + static_cast<size_t>(tok) * (p.S * p.I) + f
                                        : p.h_perm + static_cast<size_t>(row0 + tok) * p.I + f;
            *dst = __float2bfloat16_rn(silu_mul(va[j], vb[j]));
        } else if (MODE == G2_STREAM) {
            if (shared) {
                p.y_sh[static_cast<size_t>(tok) * p.H + f] = va[j];
            } else if (p.y_bf16) {
                reinterpret_cast<__nv_bfloat16*>(p.y_perm)[static_cast<size_t>(row0 + tok) * p.H + f] =
                    __float2bfloat16_rn(va[j]);
            } else {
                reinterpret_cast<float*>(p.y_perm)[static_cast<size_t>(row0 + tok) * p.H + f] = va[j];
            }
        } else {
            p.logits[static_cast<size_t>(tok) * p.V + f] = __float2bfloat16_rn(va[j]);
        }
    }
}

// ------------------------------------------------------------ host helpers (expert_ffn.cu)
// bf16 tensor [d2][d1][d0] (d0 innermost) as a rank-3 TMA map with box {64, box_rows, 1}, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint32_t box_rows);
// Packed weight tensor (moe_pack_weights layout) [n][rows][cols] as a TMA map of 16 KB tiles.
bool make_packed_map(CUtensorMap* m, const void* base, int rows, int cols, int n);
// 1 unless MOESPEC_NO_EVICT_FIRST=1.
int evict_first_allowed();
// The per-CTA device timeline buffer set by ms_set_device_trace (or null).
uint64_t* device_trace();
// Token-operand width of the streaming schedule: T rounded up to 16, 32, 64 or 128.
int stream_nmax(int T);

}  // namespace ms

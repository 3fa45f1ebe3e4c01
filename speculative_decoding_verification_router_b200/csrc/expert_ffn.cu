// a3 (and a5): grouped SwiGLU expert GEMMs on the 5th-generation tensor cores.
//
// One persistent, warp-specialised kernel template serves every contraction
// of the layer: GEMM1 (gate/up projections + SwiGLU), GEMM2 (down
// projection) and the vocab head.  Warp 0 issues TMA loads (128-byte
// swizzled tiles, no multicast), warp 1 issues tcgen05.mma from one thread
// into TMEM accumulators (two buffers, so the epilogue of one tile overlaps
// the main loop of the next), warps 2..5 drain TMEM with tcgen05.ld.
//
// Two schedules:
//  * streaming (verify-sized T <= 128): the weights are the M = 128 operand
//    and the tokens of one expert the N operand (N = rows rounded up to 16).
//    Every CTA takes the same number of whole output tiles, all but the last
//    round; the k-steps of the remaining tiles are divided into contiguous
//    ranges, one per CTA, of equal cost (weight bytes plus token-box bytes),
//    so every SM moves the same amount of data ("stream-K").  Weight tiles
//    are loaded with an L2 evict-first policy.  A CTA's part of a split tile
//    goes to an fp32 partial slot; ffn_finish_kernel, launched after the
//    GEMM, sums the two to four parts of each split tile in CTA order
//    (deterministic, no CTA ever waits on another) and applies the epilogue.
//    For GEMM1 the gate and up rows of the same 128 features accumulate into
//    two TMEM buffers in the same lanes, so SwiGLU is done in registers.
//  * tiled (prefill-sized T): the tokens of one expert are the M = 128
//    operand and the weights the N operand; for GEMM1 the N = 256 tile is
//    128 gate rows followed by the matching 128 up rows, so each thread holds
//    both halves of its token row and applies SwiGLU in registers.  GEMM2
//    runs 256 x 256 tiles on CTA pairs (ffn_gemm_pair_kernel).
// Shared experts form one extra group whose intermediate width is S*I: two
// SwiGLU experts equal one expert with the intermediates concatenated.
#include "ffn_core.cuh"
#include "layer_fused.cuh"

#include <algorithm>

namespace ms {

using namespace sm100;

// ------------------------------------------------------------ router epilogue
// Softmax over the E logits of token t and its k largest (larger logit first,
// equal logits to the lower expert), in registers: one pass keeps the k best in
// descending order.  Gate weight = softmax probability, divided by the sum of
// the k chosen when renormalising.
constexpr int ROUTE_TC_EMAX = 64;
constexpr int ROUTE_TC_KMAX = 8;

// The router's epilogue for one token row (this thread's TMEM lane), in
// registers only: in this kernel shared memory takes nearly all of L1, so a
// per-thread array indexed at run time would live in L2.  Two passes over the
// logits in chunks of 16, reloaded from TMEM: the maximum and the 8 best (kept
// in descending order, a later expert never passing an equal earlier one; the
// first k are the top-k), then the softmax denominator.  Every lane executes the TMEM
// loads (warp-collective); only a valid row stores.
template <typename TmemAt>
__device__ __forceinline__ void route_chunk(const Params& p, TmemAt tmem_at, int c16, int t, bool valid,
                                            float (&z)[16]) {
    float h16[16], m16[16], l16[16];
    tmem_ld16(tmem_at(c16 * 16), h16);
    tmem_ld16(tmem_at(p.E + c16 * 16), m16);
    tmem_ld16(tmem_at(2 * p.E + c16 * 16), l16);
    tmem_ld_wait();
#pragma unroll
    for (int j = 0; j < 16; ++j) z[j] = (h16[j] + m16[j]) + l16[j];
    if (p.rbias && valid) {
        const float* b = p.rbias + static_cast<size_t>(t) * p.E + c16 * 16;
#pragma unroll
        for (int j = 0; j < 16; ++j) z[j] += __ldg(b + j);
    }
}

template <typename TmemAt>
__device__ __forceinline__ void route_epilogue(const Params& p, TmemAt tmem_at, int t, bool valid) {
    const int E = p.E, k = p.k;
    float tv[ROUTE_TC_KMAX];   // the 8 best so far, descending (ti < 0: empty); the first k are the top-k
    int ti[ROUTE_TC_KMAX];
#pragma unroll
    for (int j = 0; j < ROUTE_TC_KMAX; ++j) {
        tv[j] = -INFINITY;
        ti[j] = -1;
    }
    float m = -INFINITY;
#pragma unroll 1
    for (int c16 = 0; c16 * 16 < E; ++c16) {
        float z[16];
        route_chunk(p, tmem_at, c16, t, valid, z);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            m = fmaxf(m, z[jj]);
            // bubble (z, e) into the list of the 8 best, ordered by logit
            // descending, then expert ascending: at each place the first of
            // the carried and the held entry in that order stays (a displaced
            // entry carries on with the same comparison)
            float cv = z[jj];
            int ci = c16 * 16 + jj;
#pragma unroll
            for (int j = 0; j < ROUTE_TC_KMAX; ++j) {
                const bool take = ti[j] < 0 || cv > tv[j] || (cv == tv[j] && ci < ti[j]);
                const float hv = tv[j];
                const int hi = ti[j];
                tv[j] = take ? cv : hv;
                ti[j] = take ? ci : hi;
                cv = take ? hv : cv;
                ci = take ? hi : ci;
            }
        }
    }
    float s = 0.f;
#pragma unroll 1
    for (int c16 = 0; c16 * 16 < E; ++c16) {
        float z[16];
        route_chunk(p, tmem_at, c16, t, valid, z);
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) s += expf(z[jj] - m);
    }
    if (!valid) return;
    float psum = 0.f;
#pragma unroll
    for (int j = 0; j < ROUTE_TC_KMAX; ++j)
        if (j < k) {
            tv[j] = expf(tv[j] - m) / s;
            psum += tv[j];
        }
#pragma unroll
    for (int j = 0; j < ROUTE_TC_KMAX; ++j)
        if (j < k) {
            p.ridx[static_cast<size_t>(t) * k + j] = ti[j];
            p.rw[static_cast<size_t>(t) * k + j] = p.rrenorm ? tv[j] / psum : tv[j];
        }
}

// ------------------------------------------------------------ kernel
template <int MODE, int NMAX>
__global__ void __launch_bounds__(NTHREADS, 1)
    ffn_gemm_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p) {
    using L = Layout<MODE, NMAX>;
    constexpr bool kStream = Cfg<MODE>::kStream;
    constexpr int kSub = Cfg<MODE>::kSub;
    // vocab head with the fused argmax: tokens are the MMA's M operand, vocabulary rows its N
    // (only with a 128-token operand; with fewer tokens the fused argmax keeps the vocabulary rows in M)
    const bool tokM = MODE == LM_STREAM && p.amax_key != nullptr && NMAX == BM;
    const bool vocM = MODE == LM_STREAM && p.amax_key != nullptr && NMAX < BM;
    constexpr bool kG1 = Cfg<MODE>::kG1;
    constexpr int ST = L::STAGES;

    extern __shared__ uint8_t dsmem[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar_full[ST], bar_empty[ST], bar_tfull[2], bar_tempty[2], bar_drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int drain_fail_sh;   // a drain wait ran out: TMEM may still be in use
    __shared__ int go_sh[2];
    __shared__ Sched sched;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = smem_addr(smem);
    const int c = blockIdx.x, nct = gridDim.x;
    const uint64_t lim = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        tstamp(p, MODE, TS_ENTRY);
        tma_prefetch_map(&maps.w_a);
        tma_prefetch_map(&maps.w_s);
        tma_prefetch_map(&maps.tok_r);
        tma_prefetch_map(&maps.tok_s);
        for (int i = 0; i < ST; ++i) {
            mbar_init(smem_addr(&bar_full[i]), 1);
            mbar_init(smem_addr(&bar_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_addr(&bar_tfull[i]), 1);
            mbar_init(smem_addr(&bar_tempty[i]), 4);
        }
        mbar_init(smem_addr(&bar_drain), 1);
        abort_sh = 0;
        drain_fail_sh = 0;
        fence_mbar_init();
    }
    // The schedule needs only the routing offsets.  They were written two or
    // more kernels back on this stream (the permutation, before the gather
    // kernel or GEMM1's finish that precedes this launch), which every kernel
    // in between waited for, so they are complete.
    build_schedule<MODE>(p, sched);
    if (threadIdx.x == 0) tstamp(p, MODE, TS_SCHEDULE);

    // ---- producer state (thread 0), kept across the dependency wait
    const int kt_h = p.H / BK, kt_i = p.I / BK;
    int q_issued = 0;                       // k-steps whose loads were issued
    int npre = 0;                           // k-steps whose weight half was prefetched
    // streaming: every weight byte is read once per launch, so its lines go
    // first when L2 needs room
    const bool hint = kStream && p.weights_evict_first;
    const uint64_t wpol = hint ? l2_policy_evict_first() : 0;
    auto weight_loads = [&](const Work& w, int kt, uint32_t a, uint32_t b, uint32_t full) {
        auto ld = [&](uint32_t dst, const CUtensorMap* m, int y, int z) {
            if (hint) tma_load_3d_hint(dst, m, full, 0, y, z, wpol);
            else tma_load_3d(dst, m, full, 0, y, z);
        };
        const bool shared = p.offsets != nullptr && w.g == p.E;
        const int kx = kt * BK;
        if (MODE == G1_STREAM || MODE == G1_TILED) {
            int z = w.g, fl = w.n * BM;
            const CUtensorMap* wm = &maps.w_a;
            if (shared) { z = fl / p.I; fl -= z * p.I; wm = &maps.w_s; }
            const uint32_t dst = MODE == G1_STREAM ? a : b;
            ld(dst, wm, packed_row(fl, kt, kt_h), z);
            ld(dst + TILE_BYTES, wm, packed_row(p.I + fl, kt, kt_h), z);
        } else if (MODE == G2_STREAM) {
            const int f0 = w.n * BM;
#pragma unroll
            for (int sb = 0; sb < kSub; ++sb) {
                const int kb = kt * kSub + sb, kxb = kb * BK;
                if (shared) {
                    const int z = kxb / p.I;
                    ld(a + sb * TILE_BYTES, &maps.w_s, packed_row(f0, (kxb - z * p.I) / BK, kt_i), z);
                } else {
                    ld(a + sb * TILE_BYTES, &maps.w_a, packed_row(f0, kb, kt_i), w.g);
                }
            }
        } else if (MODE == LM_STREAM) {
#pragma unroll
            for (int sb = 0; sb < kSub; ++sb)
                ld(a + sb * TILE_BYTES, &maps.w_a, packed_row(w.n * BM, kt * kSub + sb, kt_h), 0);
        } else if (MODE == ROUTE_TILED) {
            // the three bf16 parts of the router weights, [3E][H] row-major: k offset in x
            tma_load_3d(b, &maps.w_a, full, kx, 0, 0);
        } else {   // G2_TILED
            const int n0 = w.n * p.bn;
            for (int j = 0; j < p.bn / BM; ++j) {
                if (shared) {
                    const int z = kx / p.I;
                    ld(b + j * TILE_BYTES, &maps.w_s, packed_row(n0 + j * BM, (kx - z * p.I) / BK, kt_i), z);
                } else {
                    ld(b + j * TILE_BYTES, &maps.w_a, packed_row(n0 + j * BM, kt, kt_i), w.g);
                }
            }
        }
    };
    auto weight_bytes = [&]() -> uint32_t {
        if (MODE == G1_STREAM || MODE == G1_TILED) return 2 * TILE_BYTES;
        if (MODE == G2_TILED || MODE == ROUTE_TILED) return p.bn * BK * 2;
        return kSub * TILE_BYTES;
    };
    auto token_loads = [&](const Work& w, int kt, uint32_t a, uint32_t b, uint32_t full) -> uint32_t {
        const bool shared = p.offsets != nullptr && w.g == p.E;
        const CUtensorMap* tm = shared ? &maps.tok_s : &maps.tok_r;
        const int row0 = sched.row0[w.g];
        if (kStream) {
            // token-major argmax mode: the tokens are the M = 128 operand, all 128 rows
            const int nb = tokM ? BM / TOKBOX : (sched.rows[w.g] + TOKBOX - 1) / TOKBOX;
            mbar_expect_tx(full, kSub * nb * TOKBOX * BK * 2);
#pragma unroll
            for (int sb = 0; sb < kSub; ++sb)
                for (int j = 0; j < nb; ++j)
                    tma_load_3d(b + sb * NMAX * BK * 2 + j * TOKBOX * BK * 2, tm, full, (kt * kSub + sb) * BK,
                                row0 + j * TOKBOX, 0);
        } else {
            mbar_expect_tx(full, TILE_BYTES);
            tma_load_3d(a, tm, full, kt * BK, row0 + w.m0, 0);
        }
        return 0;
    };

    if (threadIdx.x == 0) {
        // Weight tiles do not depend on the previous kernel: start streaming
        // the first stages now, while it drains.  (Prefetching further
        // k-steps into L2 as well measured slower: the extra requests delay
        // the ones the pipeline waits for.)  The router's split weights are
        // the exception: the launch just before writes them.
        WorkIter<MODE> it;
        it.init(p, sched, c, nct);
        Work w;
        while (MODE != ROUTE_TILED && npre < ST && it.next(p, sched, w)) {
            for (int i = w.k0; i < w.k1 && npre < ST; ++i, ++npre) {
                const uint32_t a = sbase + npre * L::STAGE, full = smem_addr(&bar_full[npre]);
                mbar_expect_tx_only(full, weight_bytes());
                weight_loads(w, kstep_of(w, i), a, a + L::A_BYTES, full);
            }
        }
    }

    // Everything below may read what the previous kernels wrote (gathered
    // tokens, the previous GEMM's output) or overwrite what they still read,
    // and TMEM is only taken once the previous kernel has released it.
    grid_dep_wait();
    if (warp == 1) {
        tmem_alloc(smem_addr(&tmem_base_sh), TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_dep_launch();
    const uint32_t tmem_base = tmem_base_sh;
    if (threadIdx.x == 0) tstamp(p, MODE, TS_SETUP);

    if (warp == 0) {
      if (lane == 0) {
        // ---------------------------------------------------- TMA producer (one thread)
        bool ok = true;
        WorkIter<MODE> it;
        it.init(p, sched, c, nct);
        Work w;
        while (ok && it.next(p, sched, w)) {
            for (int i = w.k0; i < w.k1; ++i, ++q_issued) {
                const int kt = kstep_of(w, i);
                const int stage = q_issued % ST;
                const uint32_t phase = static_cast<uint32_t>(q_issued / ST) & 1u;
                const uint32_t a = sbase + stage * L::STAGE, b = a + L::A_BYTES;
                const uint32_t full = smem_addr(&bar_full[stage]);
                if (q_issued >= npre) {
                    if (!mbar_wait(smem_addr(&bar_empty[stage]), phase ^ 1u, lim, &abort_sh)) {
                        ok = false;
                        break;
                    }
                    mbar_expect_tx_only(full, weight_bytes());
                    weight_loads(w, kt, a, b, full);
                }
                token_loads(w, kt, a, b, full);   // arrives on `full` with the token bytes
            }
        }
        if (!ok) {
            report_status(p.status, MS_ERR_TIMEOUT);
            abort_sh = 1;
        }
        // drain: every load this thread issued lands before the CTA exits.  A
        // step whose weight half was prefetched but whose token half was never
        // issued (only possible if the loop stopped early) gets its arrival so
        // that its phase can complete once the weights land.
        for (int q = q_issued; q < npre; ++q) mbar_arrive(smem_addr(&bar_full[q]));
        const int q_end = q_issued > npre ? q_issued : npre;
        for (int s2 = 0; s2 < ST && s2 < q_end; ++s2) {
            const int q_last = s2 + ((q_end - 1 - s2) / ST) * ST;
            if (!mbar_wait(smem_addr(&bar_full[s2]), static_cast<uint32_t>(q_last / ST) & 1u, lim, nullptr))
                drain_failed(p.status, drain_fail_sh);
        }
        tstamp(p, MODE, TS_PRODUCER_DONE);
      }
      __syncwarp();   // lanes 1..31 wait here so the warp reaches the final barrier converged
    } else if (warp == 1) {
      if (lane == 0) {
        // ---------------------------------------------------- MMA issuer (one thread)
        int q = 0, acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        WorkIter<MODE> it;
        it.init(p, sched, c, nct);
        Work w;
        while (ok && it.next(p, sched, w)) {
            if (!mbar_wait(smem_addr(&bar_tempty[acc]), acc_phase ^ 1u, lim, &abort_sh)) { ok = false; break; }
            tc_fence_after();
            uint32_t n_mma;
            if (tokM) n_mma = BM;
            else if (kStream) n_mma = static_cast<uint32_t>((sched.rows[w.g] + 15) / 16 * 16);
            else n_mma = MODE == G1_TILED ? 256u : static_cast<uint32_t>(p.bn);
            const uint32_t idesc = idesc_bf16_f32(BM, n_mma);
            const uint32_t d0 = tmem_base + acc * 256;
            for (int kt = w.k0; kt < w.k1; ++kt, ++q) {
                const int stage = q % ST;
                if (!mbar_wait(smem_addr(&bar_full[stage]), static_cast<uint32_t>(q / ST) & 1u, lim, &abort_sh)) {
                    ok = false;
                    break;
                }
                if (q == 0) tstamp(p, MODE, TS_FIRST_DATA);
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
                        if (MODE == LM_STREAM && tokM) {   // D[token][vocab row] = x . w
                            mma_bf16(d0, bd, smem_desc_sw128(a + kk * 32), idesc, accum);
                            continue;
                        }
                        mma_bf16(d0, smem_desc_sw128(a + kk * 32), bd, idesc, accum);
                        if (MODE == G1_STREAM)
                            mma_bf16(d0 + 128, smem_desc_sw128(a + TILE_BYTES + kk * 32), bd, idesc, accum);
                    }
                }
                mma_commit(smem_addr(&bar_empty[stage]));
            }
            if (!ok) break;
            mma_commit(smem_addr(&bar_tfull[acc]));
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) {
            report_status(p.status, MS_ERR_TIMEOUT);
            abort_sh = 1;
        }
        tstamp(p, MODE, TS_LAST_MMA);
        // drain: all MMAs issued by this thread complete before TMEM is freed
        mma_commit(smem_addr(&bar_drain));
        if (!mbar_wait(smem_addr(&bar_drain), 0, lim, nullptr)) drain_failed(p.status, drain_fail_sh);
      }
      __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (4 warps)
        const int q4 = warp & 3;              // TMEM lane quadrant of this warp
        const int r_in = q4 * 32 + lane;      // accumulator row held by this thread
        const int etid = threadIdx.x - 64;    // 0..127
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        const int ldh_r = p.I, ldh_s = p.S * p.I;
        auto tmem_at = [&](int col) -> uint32_t {
            return tmem_base + (static_cast<uint32_t>(q4 * 32) << 16) + static_cast<uint32_t>(acc * 256 + col);
        };
        // one finished output value of the streaming schedule (row r_in of the tile, token t)
        auto store_stream = [&](bool shared, int row0, int f, int t, float va, float vb) {
            if (MODE == G1_STREAM) {
                __nv_bfloat16* dst = shared ? p.h_sh + static_cast<size_t>(t) * ldh_s + f
                                            : p.h_perm + static_cast<size_t>(row0 + t) * ldh_r + f;
                *dst = __float2bfloat16_rn(silu_mul(va, vb));
            } else if (MODE == G2_STREAM) {
                if (shared) {
                    p.y_sh[static_cast<size_t>(t) * p.H + f] = va;
                } else if (p.y_bf16) {
                    reinterpret_cast<__nv_bfloat16*>(p.y_perm)[static_cast<size_t>(row0 + t) * p.H + f] =
                        __float2bfloat16_rn(va);
                } else {
                    reinterpret_cast<float*>(p.y_perm)[static_cast<size_t>(row0 + t) * p.H + f] = va;
                }
            } else {
                p.logits[static_cast<size_t>(t) * p.V + f] = __float2bfloat16_rn(va);
            }
        };
        WorkIter<MODE> it;
        it.init(p, sched, c, nct);
        Work w;
        while (ok && it.next(p, sched, w)) {
            if (!epi_wait(smem_addr(&bar_tfull[acc]), acc_phase, lim, &abort_sh, etid, go_sh[acc])) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int g = w.g;
            const bool shared = p.offsets != nullptr && g == p.E;
            const int rows = sched.rows[g], row0 = sched.row0[g];
            if (kStream) {
                const int slot_floats = BM * NMAX * (kG1 ? 2 : 1);
                const int f = w.n * BM + r_in;          // output feature of this thread
                const int nch = tokM ? BM / 16 : (rows + 15) / 16;
                const bool whole = w.k0 == 0 && w.k1 == w.kt;
                float* my_slot = nullptr;
                if (!whole) {
                    const bool first = it.sk_range_begin(c) >= w.tile_start;
                    my_slot = p.partials + static_cast<size_t>(2 * c + (first ? 0 : 1)) * slot_floats;
                }
                for (int ch = 0; ch < nch; ++ch) {
                    float va[16], vb[16];
                    tmem_ld16(tmem_at(ch * 16), va);
                    if (kG1) tmem_ld16(tmem_at(128 + ch * 16), vb);
                    tmem_ld_wait();
                    if (!whole) {
                        if (kG1 || tokM) {   // token-major: [chunk][token][16 vocabulary rows]
                            slot_store16(my_slot + slot_off<NMAX>(0, ch, r_in), va);
                            if (tokM) continue;
                            slot_store16(my_slot + slot_off<NMAX>(1, ch, r_in), vb);
                        } else {
#pragma unroll
                            for (int j = 0; j < 16; ++j) my_slot[slot_off_col(ch * 16 + j, r_in)] = va[j];
                        }
                        continue;
                    }
                    if (tokM) {
                        if (r_in < rows) argmax_chunk_store(p.amax_key, p.V / 16, r_in, va, w.n * (BM / 16) + ch);
                        continue;
                    }
                    if (vocM) {
#pragma unroll
                        for (int j = 0; j < 16; ++j)
                            if (ch * 16 + j < rows)
                                argmax_warp_store(p.amax_key, p.V / 16, ch * 16 + j, va[j], r_in, w.n, q4, lane);
                        continue;
                    }
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int t = ch * 16 + j;
                        if (t < rows) store_stream(shared, row0, f, t, va[j], kG1 ? vb[j] : 0.f);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&bar_tempty[acc]));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
                // a split tile's parts are summed by ffn_finish_kernel after this kernel
            } else {
                const int rr = w.m0 + r_in;                  // row within the group
                const bool valid = rr < rows;
                const size_t orow = static_cast<size_t>(shared ? rr : row0 + rr);
                if (MODE == ROUTE_TILED) {
                    // logit of expert e = (hi + mid) + lo parts, columns e, E + e, 2E + e
                    route_epilogue(p, tmem_at, rr, valid);
                } else if (MODE == G1_TILED) {
                    const int f0 = w.n * BM;
                    __nv_bfloat16* dst = shared ? p.h_sh + orow * ldh_s + f0 : p.h_perm + orow * ldh_r + f0;
                    for (int ch = 0; ch < BM / 16; ++ch) {
                        float g16[16], u16[16];
                        tmem_ld16(tmem_at(ch * 16), g16);
                        tmem_ld16(tmem_at(128 + ch * 16), u16);
                        tmem_ld_wait();
                        if (valid) {
                            __align__(16) __nv_bfloat162 hb[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j)
                                hb[j] = __floats2bfloat162_rn(silu_mul(g16[2 * j], u16[2 * j]),
                                                              silu_mul(g16[2 * j + 1], u16[2 * j + 1]));
                            uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 16);
                            d4[0] = reinterpret_cast<const uint4*>(hb)[0];
                            d4[1] = reinterpret_cast<const uint4*>(hb)[1];
                        }
                    }
                } else {
                    const int n0 = w.n * p.bn;
                    for (int ch = 0; ch < p.bn / 16; ++ch) {
                        float v16[16];
                        tmem_ld16(tmem_at(ch * 16), v16);
                        tmem_ld_wait();
                        if (!valid) continue;
                        if (shared || !p.y_bf16) {
                            float* dst = shared ? p.y_sh + orow * p.H + n0 + ch * 16
                                                : reinterpret_cast<float*>(p.y_perm) + orow * p.H + n0 + ch * 16;
                            float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                d4[j] = make_float4(v16[4 * j], v16[4 * j + 1], v16[4 * j + 2], v16[4 * j + 3]);
                        } else {
                            __align__(16) __nv_bfloat162 hb[8];
#pragma unroll
                            for (int j = 0; j < 8; ++j) hb[j] = __floats2bfloat162_rn(v16[2 * j], v16[2 * j + 1]);
                            uint4* d4 = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.y_perm) +
                                                                 orow * p.H + n0 + ch * 16);
                            d4[0] = reinterpret_cast<const uint4*>(hb)[0];
                            d4[1] = reinterpret_cast<const uint4*>(hb)[1];
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(smem_addr(&bar_tempty[acc]));
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
        }
        if (!ok) {
            if (etid == 0) report_status(p.status, MS_ERR_TIMEOUT);
            abort_sh = 1;
        }
        if (etid == 0) tstamp(p, MODE, TS_EPI_DONE);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    // After a drain wait that ran out, loads or MMAs of this CTA may still be
    // in flight: its TMEM is left allocated rather than handed to another CTA
    // while an MMA may still write it (MS_ERR_DRAIN_TIMEOUT is recorded; the
    // device is then in an undefined state and the caller must reset it).
    if (warp == 1 && !drain_fail_sh) tmem_dealloc(tmem_base, TMEM_COLS);
    if (threadIdx.x == 32) tstamp(p, MODE, TS_EXIT);
}

// ------------------------------------------------------------ tiled GEMMs on CTA pairs
// The prefill contractions as 256 x 256 tiles on a pair of CTAs (a cluster of
// two, tcgen05 cta_group::2).  Each CTA stages 128 token rows and its half of
// the tile's 256 weight rows (GEMM1: CTA 0 the gate rows, CTA 1 the up rows of
// the same 128 features; GEMM2: 128 of the 256 output features), so a CTA
// pulls 32 KB per 64-wide k-step instead of 48 KB and keeps six stages in
// flight; the first CTA issues one M = 256, N = 256 MMA per 16-wide k-slice
// and each CTA's TMEM receives its 128 token rows x 256 columns.
//   - both CTAs' loads complete on CTA 0's `full` barrier (armed by CTA 0
//     for the pair's bytes), on which CTA 0's MMA thread waits; it commits
//     each completion twice, to `empty` (stage free) and `tfull` (accumulator
//     ready) of CTA 0 and of CTA 1, by cluster address;
//   - both CTAs' epilogue warps arrive on CTA 0's `tempty` (count 8).
// No multicast of any kind: every load reads this GPU's memory into its own CTA.
constexpr int PAIR_STAGE = 2 * TILE_BYTES;   // 128 token rows + 128 weight rows, 64 wide
constexpr int PAIR_ST = 6;
constexpr int PAIR_SMEM = PAIR_ST * PAIR_STAGE + 1024;

template <int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
    ffn_gemm_pair_kernel(const __grid_constant__ Maps maps, const __grid_constant__ Params p) {
    static_assert(MODE == G1_TILED || MODE == G2_TILED, "CTA pairs run the tiled schedule");
    constexpr int ST = PAIR_ST;
    extern __shared__ uint8_t dsmem[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(dsmem) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(8) uint64_t bar_full[ST], bar_empty[ST], bar_tfull[2], bar_tempty[2], bar_drain;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ volatile int drain_fail_sh;   // a drain wait ran out: TMEM may still be in use
    __shared__ int go_sh[2];
    __shared__ Sched sched;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t sbase = smem_addr(smem);
    const uint32_t rank = cluster_rank();          // 0: issues the MMAs
    const int pc = static_cast<int>(blockIdx.x >> 1), npair = static_cast<int>(gridDim.x >> 1);
    const uint64_t lim = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        tstamp(p, MODE, TS_ENTRY);
        tma_prefetch_map(&maps.w_a);
        tma_prefetch_map(&maps.w_s);
        tma_prefetch_map(&maps.tok_r);
        tma_prefetch_map(&maps.tok_s);
        for (int i = 0; i < ST; ++i) {
            mbar_init(smem_addr(&bar_full[i]), 1);
            mbar_init(smem_addr(&bar_empty[i]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_addr(&bar_tfull[i]), 1);
            mbar_init(smem_addr(&bar_tempty[i]), 8);
        }
        mbar_init(smem_addr(&bar_drain), 1);
        abort_sh = 0;
        drain_fail_sh = 0;
        fence_mbar_init();
    }
    build_schedule<MODE>(p, sched);
    grid_dep_wait();
    // both CTAs' barriers exist before either CTA signals the other's
    cluster_sync_all();
    if (warp == 1) {
        tmem_alloc_pair(smem_addr(&tmem_base_sh), TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_dep_launch();
    const uint32_t tmem_base = tmem_base_sh;
    if (threadIdx.x == 0) tstamp(p, MODE, TS_SETUP);
    const int kt_h = p.H / BK, kt_i = p.I / BK;

    if (warp == 0) {
      if (lane == 0) {
        // ---------------------------------------------------- TMA producer (this CTA's halves)
        bool ok = true;
        int q = 0;
        const uint32_t full0 = mapa_shared(smem_addr(&bar_full[0]), 0);
        WorkIter<MODE> it;
        it.init(p, sched, pc, npair);
        Work w;
        while (ok && it.next(p, sched, w)) {
            const bool shared = p.offsets != nullptr && w.g == p.E;
            const CUtensorMap* tm = shared ? &maps.tok_s : &maps.tok_r;
            const int trow = sched.row0[w.g] + w.m0 + static_cast<int>(rank) * BM;
            for (int kt = w.k0; kt < w.k1; ++kt, ++q) {
                const int stage = q % ST;
                const uint32_t phase = static_cast<uint32_t>(q / ST) & 1u;
                if (!mbar_wait(smem_addr(&bar_empty[stage]), phase ^ 1u, lim, &abort_sh)) {
                    ok = false;
                    break;
                }
                const uint32_t a = sbase + stage * PAIR_STAGE, b = a + TILE_BYTES;
                // both CTAs' loads complete on CTA 0's `full` barrier, which
                // CTA 0's producer arms for the pair's 64 KB
                const uint32_t full = full0 + stage * 8;
                if (rank == 0) mbar_expect_tx(smem_addr(&bar_full[stage]), 2 * PAIR_STAGE);
                tma_load_3d_pair(a, tm, full, kt * BK, trow, 0);
                if (MODE == G1_TILED) {
                    int z = w.g, fl = w.n * BM;
                    const CUtensorMap* wm = &maps.w_a;
                    if (shared) { z = fl / p.I; fl -= z * p.I; wm = &maps.w_s; }
                    tma_load_3d_pair(b, wm, full, 0, packed_row(rank == 0 ? fl : p.I + fl, kt, kt_h), z);
                } else {
                    const int n0 = w.n * 2 * BM + static_cast<int>(rank) * BM;
                    if (shared) {
                        const int kx = kt * BK, z = kx / p.I;
                        tma_load_3d_pair(b, &maps.w_s, full, 0, packed_row(n0, (kx - z * p.I) / BK, kt_i), z);
                    } else {
                        tma_load_3d_pair(b, &maps.w_a, full, 0, packed_row(n0, kt, kt_i), w.g);
                    }
                }
            }
        }
        if (!ok) {
            report_status(p.status, MS_ERR_TIMEOUT);
            abort_sh = 1;
        }
        // drain: every load this thread issued has landed once CTA 0's MMAs
        // released its stage (they waited for the full pair of loads)
        for (int s2 = 0; s2 < ST && s2 < q; ++s2) {
            const int q_last = s2 + ((q - 1 - s2) / ST) * ST;
            if (!mbar_wait(smem_addr(&bar_empty[s2]), static_cast<uint32_t>(q_last / ST) & 1u, lim, nullptr))
                drain_failed(p.status, drain_fail_sh);
        }
        tstamp(p, MODE, TS_PRODUCER_DONE);
      }
      __syncwarp();
    } else if (warp == 1) {
      if (lane == 0) {
        if (rank == 0) {
            bool ok = true;
            WorkIter<MODE> it;
            it.init(p, sched, pc, npair);
            Work w;
            // ---------------------------------------------------- MMA issuer (one thread of CTA 0)
            const uint32_t idesc = idesc_bf16_f32(2 * BM, 2 * BM);
            // each completion is committed to this CTA's barrier and to the peer's
            const uint32_t empty_self = mapa_shared(smem_addr(&bar_empty[0]), 0);
            const uint32_t empty_peer = mapa_shared(smem_addr(&bar_empty[0]), 1);
            const uint32_t tfull_self = mapa_shared(smem_addr(&bar_tfull[0]), 0);
            const uint32_t tfull_peer = mapa_shared(smem_addr(&bar_tfull[0]), 1);
            int q = 0, acc = 0;
            uint32_t acc_phase = 0;
            while (ok && it.next(p, sched, w)) {
                if (!mbar_wait(smem_addr(&bar_tempty[acc]), acc_phase ^ 1u, lim, &abort_sh)) { ok = false; break; }
                tc_fence_after();
                const uint32_t d0 = tmem_base + acc * 256;
                for (int kt = w.k0; kt < w.k1; ++kt, ++q) {
                    const int stage = q % ST;
                    const uint32_t phase = static_cast<uint32_t>(q / ST) & 1u;
                    if (!mbar_wait(smem_addr(&bar_full[stage]), phase, lim, &abort_sh)) {
                        ok = false;
                        break;
                    }
                    if (q == 0) tstamp(p, MODE, TS_FIRST_DATA);
                    tc_fence_after();
                    const uint32_t a = sbase + stage * PAIR_STAGE, b = a + TILE_BYTES;
#pragma unroll
                    for (int kk = 0; kk < BK / 16; ++kk)
                        mma_bf16_pair(d0, smem_desc_sw128(a + kk * 32), smem_desc_sw128(b + kk * 32), idesc,
                                      (kt > w.k0 || kk > 0) ? 1u : 0u);
                    mma_commit_pair(empty_self + stage * 8);
                    mma_commit_pair(empty_peer + stage * 8);
                }
                if (!ok) break;
                mma_commit_pair(tfull_self + acc * 8);
                mma_commit_pair(tfull_peer + acc * 8);
                acc ^= 1;
                if (acc == 0) acc_phase ^= 1u;
            }
            if (!ok) {
                report_status(p.status, MS_ERR_TIMEOUT);
                abort_sh = 1;
            }
            tstamp(p, MODE, TS_LAST_MMA);
            // drain: every pair MMA issued by this thread completes before TMEM is freed
            mma_commit_pair(mapa_shared(smem_addr(&bar_drain), 0));
            if (!mbar_wait(smem_addr(&bar_drain), 0, lim, nullptr)) drain_failed(p.status, drain_fail_sh);
        }
      }
      __syncwarp();
    } else {
        // ---------------------------------------------------- epilogue (4 warps, this CTA's 128 rows)
        const int q4 = warp & 3;
        const int r_in = q4 * 32 + lane;
        const int etid = threadIdx.x - 64;
        int acc = 0;
        uint32_t acc_phase = 0;
        bool ok = true;
        const int ldh_r = p.I, ldh_s = p.S * p.I;
        const uint32_t tempty0 = mapa_shared(smem_addr(&bar_tempty[0]), 0);
        auto tmem_at = [&](int col) -> uint32_t {
            return tmem_base + (static_cast<uint32_t>(q4 * 32) << 16) + static_cast<uint32_t>(acc * 256 + col);
        };
        WorkIter<MODE> it;
        it.init(p, sched, pc, npair);
        Work w;
        while (ok && it.next(p, sched, w)) {
            if (!epi_wait(smem_addr(&bar_tfull[acc]), acc_phase, lim, &abort_sh, etid, go_sh[acc])) {
                ok = false;
                break;
            }
            tc_fence_after();
            const int g = w.g;
            const bool shared = p.offsets != nullptr && g == p.E;
            const int rows = sched.rows[g], row0 = sched.row0[g];
            const int rr = w.m0 + static_cast<int>(rank) * BM + r_in;   // row within the group
            const bool valid = rr < rows;
            const size_t orow = static_cast<size_t>(shared ? rr : row0 + rr);
            if (MODE == G1_TILED) {
                const int f0 = w.n * BM;
                __nv_bfloat16* dst = shared ? p.h_sh + orow * ldh_s + f0 : p.h_perm + orow * ldh_r + f0;
                for (int ch = 0; ch < BM / 16; ++ch) {
                    float g16[16], u16[16];
                    tmem_ld16(tmem_at(ch * 16), g16);
                    tmem_ld16(tmem_at(128 + ch * 16), u16);
                    tmem_ld_wait();
                    if (valid) {
                        __align__(16) __nv_bfloat162 hb[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            hb[j] = __floats2bfloat162_rn(silu_mul(g16[2 * j], u16[2 * j]),
                                                          silu_mul(g16[2 * j + 1], u16[2 * j + 1]));
                        uint4* d4 = reinterpret_cast<uint4*>(dst + ch * 16);
                        d4[0] = reinterpret_cast<const uint4*>(hb)[0];
                        d4[1] = reinterpret_cast<const uint4*>(hb)[1];
                    }
                }
            } else {
                const int n0 = w.n * 2 * BM;
                for (int ch = 0; ch < 2 * BM / 16; ++ch) {
                    float v16[16];
                    tmem_ld16(tmem_at(ch * 16), v16);
                    tmem_ld_wait();
                    if (!valid) continue;
                    if (shared || !p.y_bf16) {
                        float* dst = shared ? p.y_sh + orow * p.H + n0 + ch * 16
                                            : reinterpret_cast<float*>(p.y_perm) + orow * p.H + n0 + ch * 16;
                        float4* d4 = reinterpret_cast<float4*>(dst);
#pragma unroll
                        for (int j = 0; j < 4; ++j)
                            d4[j] = make_float4(v16[4 * j], v16[4 * j + 1], v16[4 * j + 2], v16[4 * j + 3]);
                    } else {
                        __align__(16) __nv_bfloat162 hb[8];
#pragma unroll
                        for (int j = 0; j < 8; ++j) hb[j] = __floats2bfloat162_rn(v16[2 * j], v16[2 * j + 1]);
                        uint4* d4 = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(p.y_perm) +
                                                             orow * p.H + n0 + ch * 16);
                        d4[0] = reinterpret_cast<const uint4*>(hb)[0];
                        d4[1] = reinterpret_cast<const uint4*>(hb)[1];
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
                if (rank == 0) mbar_arrive(smem_addr(&bar_tempty[acc]));
                else mbar_arrive_remote(tempty0 + acc * 8);
            }
            acc ^= 1;
            if (acc == 0) acc_phase ^= 1u;
        }
        if (!ok) {
            if (etid == 0) report_status(p.status, MS_ERR_TIMEOUT);
            abort_sh = 1;
        }
        if (etid == 0) tstamp(p, MODE, TS_EPI_DONE);
    }
    tc_fence_before();
    __syncthreads();
    // CTA 0's last MMAs read this CTA's shared memory and write its TMEM: neither
    // CTA frees either before both got here
    cluster_sync_all();
    tc_fence_after();
    // the pair's TMEM is released by both CTAs together, and only if neither
    // CTA's drain wait ran out (see ffn_gemm_kernel)
    if (warp == 1 && !drain_fail_sh && !peer_flag(&drain_fail_sh)) tmem_dealloc_pair(tmem_base, TMEM_COLS);
    if (threadIdx.x == 32) tstamp(p, MODE, TS_EXIT);
}

template <int MODE, int NMAX>
// After the gate/up GEMM at 32+ tokens the kernel is held to three CTAs' worth of
// registers per SM: two of its CTAs and the down GEMM's CTA then share an SM.
__global__ void __launch_bounds__(FIN_THREADS, (MODE == G1_STREAM && NMAX >= 32) ? 3 : 1) ffn_finish_kernel(const __grid_constant__ Params p) {
    __shared__ Sched sched;
    __shared__ int iprefix[MAX_GROUPS + 1];   // items before group g
    fin_stamp<MODE>(p, TS_ENTRY);
    // The offsets come from a kernel at least two launches back, which every
    // kernel of this library waits for before it lets its successor start:
    // they may be read before this launch's own wait.
    build_schedule_n<MODE, FIN_THREADS>(p, sched);
    const bool tokM = MODE == LM_STREAM && p.amax_key != nullptr && NMAX == BM;
    const int ng = sched.ngroups;
    const int nt = sched.tprefix[ng];
    const int first_split = p.nct * dp_tiles_per_cta(nt, p.nct);
    auto nchunks = [&](int g) { return tokM ? BM / 16 : (sched.rows[g] + 15) / 16; };
    // with at most 16 tokens every split tile is one item: item i is split tile i
    constexpr bool kOneChunk = NMAX == 16;
    if (!kOneChunk) {
        for (int g = threadIdx.x; g < ng; g += FIN_THREADS) {
            const int lo = max(first_split, sched.tprefix[g]), hi = sched.tprefix[g + 1];
            iprefix[g + 1] = hi > lo ? (hi - lo) * nchunks(g) : 0;
        }
        __syncthreads();
        if (threadIdx.x < 32) warp_scan_groups(iprefix, ng, threadIdx.x);
        __syncthreads();
    }
    const int nitems = kOneChunk ? nt - first_split : iprefix[ng];
    grid_dep_wait();
    grid_dep_launch();
    fin_stamp<MODE>(p, TS_SCHEDULE);
    WorkIter<MODE> it;
    it.init(p, sched, 0, p.nct);
    if constexpr (kOneChunk) {
        // the grid (2 nct CTAs) covers every split tile: one item per CTA, no
        // loop (a loop around the item doubles the kernel's register use)
        const int item = static_cast<int>(blockIdx.x);
        if (item < nitems) {
            const int t = first_split + item;
            finish_item<MODE, NMAX>(p, sched, it, find_group_tile(sched, t), t, 0);
        }
    } else {
#pragma unroll 1
        for (int item = static_cast<int>(blockIdx.x); item < nitems; item += static_cast<int>(gridDim.x)) {
            // group of the item: largest g with iprefix[g] <= item (groups
            // without items have iprefix[g] == iprefix[g + 1] and are never chosen)
            int lo = 0, hi = ng - 1;
            while (lo < hi) {
                const int mid = (lo + hi + 1) >> 1;
                if (iprefix[mid] <= item) lo = mid; else hi = mid - 1;
            }
            const int g = lo;
            const int nch = nchunks(g);
            const int local = item - iprefix[g];
            finish_item<MODE, NMAX>(p, sched, it, g, max(first_split, sched.tprefix[g]) + local / nch,
                                    local - (local / nch) * nch);
        }
    }
    fin_stamp<MODE>(p, TS_EXIT);
}

// ------------------------------------------------------------ prep kernel
// Gathers the routed token rows into expert order, pads token operands to
// whole TMA boxes with zeros.
__global__ void __launch_bounds__(256) ffn_prep_kernel(const __nv_bfloat16* __restrict__ x,
                                                       const int32_t* __restrict__ perm, int T,
                                                       int H, int rows, int rows_pad,
                                                       __nv_bfloat16* __restrict__ x_perm,
                                                       __nv_bfloat16* __restrict__ x_pad,
                                                       int t_pad, int32_t* status) {
    grid_dep_wait();
    grid_dep_launch();
    // one warp per output row: the row's token id is read once, then the warp
    // copies the row in 16-byte pieces (a 2,560-byte row is 5 per lane)
    const int lane = threadIdx.x & 31;
    const int n8 = H / 8;
    const int nwarps = gridDim.x * (blockDim.x >> 5);
    const int warp0 = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    for (int r = warp0; r < rows_pad; r += nwarps) {
        int t = -1;
        if (r < rows) {
            t = __ldg(perm + r);
            if (t < 0 || t >= T) {
                if (lane == 0) report_status(status, MS_ERR_DEVICE_INDEX);
                t = -1;
            }
        }
        const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(t < 0 ? 0 : t) * H);
        uint4* dst = reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(r) * H);
        for (int c = lane; c < n8; c += 32) dst[c] = t >= 0 ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
    if (x_pad) {
        for (int r = warp0; r < t_pad; r += nwarps) {
            const uint4* src = reinterpret_cast<const uint4*>(x + static_cast<size_t>(r < T ? r : 0) * H);
            uint4* dst = reinterpret_cast<uint4*>(x_pad + static_cast<size_t>(r) * H);
            for (int c = lane; c < n8; c += 32) dst[c] = r < T ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
        }
    }
}

// Prefill gather: x_perm[r] = x[perm[r]] for r < rows (the token rows in
// expert order), rows..rows_pad-1 zero.  CTA c copies the contiguous rows
// [c*per, (c+1)*per): their token ids are read once into shared memory, then
// one thread streams them in chunks of R rows (R*H*2 <= 20 KB) through a ring
// of GB_NS shared-memory slots -- a bulk load per row (the whole row) into the
// chunk's slot and, GB_LAG chunks later, once those loads have landed, one
// bulk store of the chunk (its rows are consecutive in x_perm).  No data
// passes through registers, so a CTA keeps GB_LAG + 1 chunks in flight; with
// two CTAs per SM that is about 120 KB per SM, where the warp-per-row kernel
// keeps one row's loads per warp and waits on each row's id first.
constexpr int GB_NS = 4, GB_LAG = 2, GB_THREADS = 128;
static_assert(GB_LAG >= 1 && GB_LAG < GB_NS, "gather ring");

__global__ void __launch_bounds__(GB_THREADS) gather_bulk_kernel(const __nv_bfloat16* __restrict__ x,
                                                                 const int32_t* __restrict__ perm, int T, int H,
                                                                 int rows, int rows_pad, int per, int R,
                                                                 __nv_bfloat16* __restrict__ x_perm,
                                                                 int32_t* status, uint64_t lim) {
    extern __shared__ __align__(128) uint8_t gsm[];
    __shared__ __align__(8) uint64_t full[GB_NS];
    const uint32_t row_bytes = static_cast<uint32_t>(H) * 2u;
    const uint32_t slot_bytes = static_cast<uint32_t>(R) * row_bytes;
    int32_t* ids = reinterpret_cast<int32_t*>(gsm + GB_NS * slot_bytes);
    const int r0 = static_cast<int>(blockIdx.x) * per;
    const int r1 = min(r0 + per, rows_pad);
    const int r1c = max(r0, min(r1, rows));   // [r0, r1c): rows with a token
    if (threadIdx.x == 0) {
        for (int i = 0; i < GB_NS; ++i) mbar_init(smem_addr(&full[i]), 1);
        fence_mbar_init();
    }
    grid_dep_wait();
    grid_dep_launch();
    // pad rows: zeros
    const int n8 = H / 8;
    for (long v = threadIdx.x; v < static_cast<long>(r1 - r1c) * n8; v += GB_THREADS)
        reinterpret_cast<uint4*>(x_perm + static_cast<size_t>(r1c) * H)[v] = make_uint4(0, 0, 0, 0);
    for (int i = threadIdx.x; i < r1c - r0; i += GB_THREADS) {
        int t = __ldg(perm + r0 + i);
        if (t < 0 || t >= T) {
            report_status(status, MS_ERR_DEVICE_INDEX);   // the row's contents are then undefined
            t = 0;
        }
        ids[i] = t;
    }
    __syncthreads();
    if (threadIdx.x != 0 || r1c == r0) return;
    const int n = (r1c - r0 + R - 1) / R;
    const uint32_t sbase = smem_addr(gsm);
    int issued = 0, stored = 0;
    bool ok = true;
    for (int i = 0; i < n + GB_LAG && ok; ++i) {
        if (i < n) {
            // the slot's previous chunk (i - GB_NS) was stored GB_NS - 1 - GB_LAG groups ago
            if (i >= GB_NS) bulk_wait_read<GB_NS - 1 - GB_LAG>();
            const int sl = i % GB_NS, nr = min(R, r1c - r0 - i * R);
            const uint32_t bar = smem_addr(&full[sl]);
            mbar_expect_tx(bar, static_cast<uint32_t>(nr) * row_bytes);
            for (int j = 0; j < nr; ++j)
                bulk_load(sbase + sl * slot_bytes + j * row_bytes, x + static_cast<size_t>(ids[i * R + j]) * H,
                          row_bytes, bar);
            issued = i + 1;
        }
        const int jd = i - GB_LAG;
        if (jd >= 0 && jd < n) {
            const int sl = jd % GB_NS, nr = min(R, r1c - r0 - jd * R);
            if (!mbar_wait(smem_addr(&full[sl]), static_cast<uint32_t>(jd / GB_NS) & 1u, lim, nullptr)) {
                report_status(status, MS_ERR_TIMEOUT);
                ok = false;
                break;
            }
            bulk_store(x_perm + static_cast<size_t>(r0 + jd * R) * H, sbase + sl * slot_bytes,
                       static_cast<uint32_t>(nr) * row_bytes);
            bulk_commit();
            stored = jd + 1;
        }
    }
    // after a timeout: the loads still in flight land before the CTA exits (bounded)
    for (int jd = stored; jd < issued; ++jd) {
        if (!mbar_wait(smem_addr(&full[jd % GB_NS]), static_cast<uint32_t>(jd / GB_NS) & 1u, lim, nullptr)) {
            report_status(status, MS_ERR_DRAIN_TIMEOUT);
            break;
        }
    }
    bulk_wait<0>();   // every store complete before the kernel ends
}

// Grid and shared memory of gather_bulk_kernel: two CTAs per SM, rows dealt in
// contiguous ranges (a multiple of the chunk).
struct GatherPlan {
    int R, per, grid;
    size_t smem;
};
static GatherPlan gather_plan(int H, int rows_pad) {
    GatherPlan g{};
    const int row_bytes = H * 2;
    g.R = 20480 / row_bytes < 1 ? 1 : (20480 / row_bytes > 8 ? 8 : 20480 / row_bytes);
    const int ctas = 2 * num_sms();
    int per = (rows_pad + ctas - 1) / ctas;
    per = (per + g.R - 1) / g.R * g.R;
    if (per > 4096) per = 4096;   // the id table stays within 16 KB
    g.per = per < g.R ? g.R : per;
    g.grid = (rows_pad + g.per - 1) / g.per;
    g.smem = static_cast<size_t>(GB_NS) * g.R * row_bytes + static_cast<size_t>(g.per) * 4;
    return g;
}

// ------------------------------------------------------------ host side
// MOESPEC_NO_EVICT_FIRST=1 loads the streamed weights with the default L2
// policy (for comparison).
int evict_first_allowed() {
    static const int on = [] {
        const char* e = getenv("MOESPEC_NO_EVICT_FIRST");
        return (e && e[0] == '1') ? 0 : 1;
    }();
    return on;
}

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// bf16 tensor [d2][d1][d0] (d0 innermost), box {64, box_rows, 1}, 128-byte swizzle.
// Every map is rank 3 (token operands use d2 = 1), so every load is the 3-D
// form of cp.async.bulk.tensor: the instruction rank must match the map.
bool make_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
              uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {d0, d1, d2};
    const cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
    const cuuint32_t box[3] = {static_cast<cuuint32_t>(BK), box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// Packed weight tensor [n][rows/128][cols/64][128][64] viewed as rank 3:
// 64-element rows, rows*cols/64 of them per matrix, n matrices.  One box of
// 64 x 128 is one contiguous 16 KB tile.
bool make_packed_map(CUtensorMap* m, const void* base, int rows, int cols, int n) {
    return make_map(m, base, BK, static_cast<uint64_t>(rows) * cols / BK, n, BM);
}

template <int MODE, int NMAX>
static ms_status launch_gemm(int id, const Maps& maps, const Params& prm, cudaStream_t s) {
    using L = Layout<MODE, NMAX>;
    static PerDevice attr;
    const int ok = attr.get([] {
        const cudaError_t e =
            cudaFuncSetAttribute(ffn_gemm_kernel<MODE, NMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, L::SMEM);
        if (e != cudaSuccess) {
            set_cuda_error(e);
            return -1;
        }
        return 1;
    });
    if (ok < 0) return MS_ERR_CUDA;
    return launch(id, ffn_gemm_kernel<MODE, NMAX>, dim3(num_sms()), dim3(NTHREADS), L::SMEM, s, maps, prm);
}

// The tiled GEMM on CTA pairs: as many pairs as can be resident at once (at
// most one CTA per SM), 0 if the device cannot place any.
template <int MODE>
static int pair_grid() {
    // cached per device as grid + 1 (a slot of 0 is empty)
    static PerDevice cache;
    return cache.get([]() -> int {
        int grid = 0;
        if (cudaFuncSetAttribute(ffn_gemm_pair_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 PAIR_SMEM) != cudaSuccess ||
            cudaFuncSetAttribute(ffn_gemm_pair_kernel<MODE>, cudaFuncAttributeNonPortableClusterSizeAllowed, 0) !=
                cudaSuccess) {
            cudaGetLastError();
            return grid + 1;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(num_sms());
        cfg.blockDim = dim3(NTHREADS);
        cfg.dynamicSmemBytes = PAIR_SMEM;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int nclusters = 0;
        if (cudaOccupancyMaxActiveClusters(&nclusters, ffn_gemm_pair_kernel<MODE>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            nclusters = 0;
        }
        const int cap = num_sms() / 2;
        grid = 2 * (nclusters < cap ? nclusters : cap);
        return grid + 1;
    }) - 1;
}

template <int MODE>
static ms_status launch_gemm_pair(int id, const Maps& maps, Params prm, cudaStream_t s) {
    prm.mt = 2 * BM;
    return launch_cluster(id, ffn_gemm_pair_kernel<MODE>, dim3(pair_grid<MODE>()), dim3(NTHREADS), PAIR_SMEM, s, 2,
                          maps, prm);
}

template <int MODE, int NMAX>
static ms_status launch_stream_n(int id, const Maps& maps, Params prm, cudaStream_t s) {
    prm.nct = num_sms();
    if (prm.nct > MAX_CTAS) return MS_ERR_UNSUPPORTED;   // the schedule keeps one range per CTA
    prm.weights_evict_first = evict_first_allowed();
    prm.invariant = batch_invariant();
    ms_status st = launch_gemm<MODE, NMAX>(id, maps, prm, s);
    if (st != MS_OK) return st;
    if (prm.invariant) return MS_OK;   // every tile whole: no split tiles to finish
    // fewer than 2 nct tiles are split; one CTA per (tile, 16-column chunk)
    return launch(K_FFN_FINISH, ffn_finish_kernel<MODE, NMAX>, dim3(finish_grid<MODE, NMAX>(prm.nct)),
                  dim3(FIN_THREADS), 0, s, prm);
}

// The streaming GEMM followed by the kernel that finishes its split tiles.
template <int MODE>
static ms_status launch_stream(int id, int nmax, const Maps& maps, const Params& prm, cudaStream_t s) {
    switch (nmax) {
        case 16: return launch_stream_n<MODE, 16>(id, maps, prm, s);
        case 32: return launch_stream_n<MODE, 32>(id, maps, prm, s);
        case 64: return launch_stream_n<MODE, 64>(id, maps, prm, s);
        default: return launch_stream_n<MODE, 128>(id, maps, prm, s);
    }
}

// MOESPEC_NO_BULK_GATHER=1 gathers the prefill token rows one warp per row (for comparison).
static bool gather_bulk_off() {
    static const bool off = [] {
        const char* e = getenv("MOESPEC_NO_BULK_GATHER");
        return e && e[0] == '1';
    }();
    return off;
}

// MOESPEC_NO_PAIR=1 runs the prefill GEMMs on single CTAs (for comparison).
static bool pair_off() {
    static int v = -1;
    if (v < 0) {
        const char* e = getenv("MOESPEC_NO_PAIR");
        v = (e && e[0] == '1') ? 1 : 0;
    }
    return v == 1;
}

static uint64_t* g_dtrace = nullptr;
void set_device_trace(void* buf) { g_dtrace = static_cast<uint64_t*>(buf); }
uint64_t* device_trace() { return g_dtrace; }

int stream_nmax(int T) {
    int n = 16;
    while (n < T) n *= 2;
    return n;
}

struct FfnWs {
    int32_t* status;
    __nv_bfloat16 *x_pad, *x_perm, *h_perm, *h_sh;
    float* partials;
    size_t bytes;
    int t_pad, rows_pad;
};

static FfnWs ffn_ws_layout(void* base, int T, int H, int E, int I, int S, int k) {
    FfnWs w{};
    char* p = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) -> char* {
        char* r = p ? p + off : nullptr;
        off += align_up(bytes, 1024);
        return r;
    };
    const bool stream = T <= 128;
    w.t_pad = static_cast<int>(align_up(T, BM));
    w.rows_pad = static_cast<int>(align_up(static_cast<size_t>(T) * k, BM));
    w.status = reinterpret_cast<int32_t*>(take(256));
    w.x_pad = reinterpret_cast<__nv_bfloat16*>(take(stream ? static_cast<size_t>(w.t_pad) * H * 2 : 0));
    w.x_perm = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(w.rows_pad) * H * 2));
    w.h_perm = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(w.rows_pad) * I * 2));
    w.h_sh = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(w.t_pad) * (S > 0 ? S * I : BK) * 2));
    const size_t slot = static_cast<size_t>(BM) * (stream ? stream_nmax(T) : 16) * 2 * sizeof(float);
    w.partials = reinterpret_cast<float*>(take(stream ? slot * 4 * num_sms() : 0));
    w.bytes = off;
    return w;
}

size_t ffn_ws_bytes(int T, int H, int E, int I, int S, int k) {
    return ffn_ws_layout(nullptr, T, H, E, I, S, k).bytes;
}

void ffn_ws_buffers(void* ws, int T, int H, int E, int I, int S, int k, LfBuffers& b) {
    const FfnWs w = ffn_ws_layout(ws, T, H, E, I, S, k);
    b.x_pad = w.x_pad;
    b.x_perm = w.x_perm;
    b.h_perm = w.h_perm;
    b.h_sh = w.h_sh;
    b.partials = w.partials;
    b.status = w.status;
    b.rows_pad = w.rows_pad;
    b.t_pad = w.t_pad;
}

ms_status ffn_launch(const void* x, const int32_t* offsets, const int32_t* perm, const void* wgu,
                     const void* wd, const void* wsgu, const void* wsd, int T, int H, int E, int I,
                     int S, int k, void* y_perm, ms_dtype ydt, float* y_sh, void* ws,
                     cudaStream_t s) {
    FfnWs w = ffn_ws_layout(ws, T, H, E, I, S, k);
    const bool stream = T <= 128;
    const int rows = T * k;
    // 1. gather + pad: prefill through the bulk-copy ring, verify sizes one warp per row
    if (!stream && w.rows_pad > 0 && !gather_bulk_off()) {
        const GatherPlan g = gather_plan(H, w.rows_pad);
        static PerDevice attr;
        const int ok = attr.get([] {
            const cudaError_t e =
                cudaFuncSetAttribute(gather_bulk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 112 * 1024);
            if (e != cudaSuccess) {
                set_cuda_error(e);
                return -1;
            }
            return 1;
        });
        if (ok < 0) return MS_ERR_CUDA;
        if (g.smem > 112 * 1024) return MS_ERR_UNSUPPORTED;
        ms_status st = launch(K_FFN_PREP, gather_bulk_kernel, dim3(g.grid), dim3(GB_THREADS), g.smem, s,
                              reinterpret_cast<const __nv_bfloat16*>(x), perm, T, H, rows, w.rows_pad, g.per, g.R,
                              w.x_perm, w.status, wait_limit_ns());
        if (st != MS_OK) return st;
    } else {
        const long want = (static_cast<long>(w.rows_pad) + 7) / 8;
        const int grid = static_cast<int>(want < 8L * num_sms() ? want : 8L * num_sms());
        ms_status st = launch(K_FFN_PREP, ffn_prep_kernel, dim3(grid), dim3(256), 0, s,
                              reinterpret_cast<const __nv_bfloat16*>(x), perm, T, H, rows, w.rows_pad,
                              w.x_perm, stream ? w.x_pad : static_cast<__nv_bfloat16*>(nullptr), w.t_pad,
                              w.status);
        if (st != MS_OK) return st;
    }
    Params prm{};
    prm.T = T; prm.H = H; prm.E = E; prm.I = I; prm.S = S; prm.k = k; prm.V = 0;
    prm.bn = (H % 256 == 0) ? 256 : 128;
    prm.offsets = offsets;
    prm.h_perm = w.h_perm;
    prm.h_sh = w.h_sh;
    prm.y_perm = y_perm;
    prm.y_bf16 = ydt == MS_BF16;
    prm.y_sh = y_sh;
    prm.partials = w.partials;
    prm.status = w.status;
    prm.wait_limit_ns = wait_limit_ns();
    prm.dtrace = g_dtrace;
    const uint32_t tok_box = stream ? TOKBOX : BM;
    const void* x_tok_s = stream ? static_cast<const void*>(w.x_pad) : x;
    const int x_rows = stream ? w.t_pad : T;
    // 2. GEMM1: gate/up + SwiGLU -> h;  3. GEMM2: down projection -> y_perm, y_shared
    Maps m1{}, m2{};
    bool ok = make_packed_map(&m1.w_a, wgu, 2 * I, H, E) &&
              make_map(&m1.tok_r, w.x_perm, H, w.rows_pad, 1, tok_box) &&
              make_map(&m1.tok_s, x_tok_s, H, x_rows, 1, tok_box);
    ok = ok && (S > 0 ? make_packed_map(&m1.w_s, wsgu, 2 * I, H, S) : make_packed_map(&m1.w_s, wgu, 2 * I, H, E));
    const int hs_cols = S > 0 ? S * I : BK;
    ok = ok && make_packed_map(&m2.w_a, wd, H, I, E) && make_map(&m2.tok_r, w.h_perm, I, w.rows_pad, 1, tok_box) &&
         make_map(&m2.tok_s, w.h_sh, hs_cols, w.t_pad, 1, tok_box);
    ok = ok && (S > 0 ? make_packed_map(&m2.w_s, wsd, H, I, S) : make_packed_map(&m2.w_s, wd, H, I, E));
    if (!ok) return MS_ERR_CUDA;
    if (stream) {
        ms_status st1 = launch_stream<G1_STREAM>(K_GEMM1_STREAM, stream_nmax(T), m1, prm, s);
        if (st1 != MS_OK) return st1;
        return launch_stream<G2_STREAM>(K_GEMM2_STREAM, stream_nmax(T), m2, prm, s);
    }
    // prefill: both GEMMs on CTA pairs, 256-token tiles.  GEMM2 (256 x 256 output
    // tiles when the output width splits in 256s): 638 vs 789 us at 36,992
    // tokens.  GEMM1 (256 tokens x 128 gate + 128 up features): 1,203-1,212 vs
    // 1,246-1,279 us; each CTA stages 32 KB per k-step instead of 48 KB, which
    // also lowers the power drawn, so the clock under the power cap is higher.
    // MOESPEC_NO_PAIR=1 runs both on single CTAs.
    ms_status st = (!pair_off() && pair_grid<G1_TILED>() >= 2)
                       ? launch_gemm_pair<G1_TILED>(K_GEMM1_TILED, m1, prm, s)
                       : launch_gemm<G1_TILED, 16>(K_GEMM1_TILED, m1, prm, s);
    if (st != MS_OK) return st;
    if (prm.bn == 256 && !pair_off() && pair_grid<G2_TILED>() >= 2)
        return launch_gemm_pair<G2_TILED>(K_GEMM2_TILED, m2, prm, s);
    return launch_gemm<G2_TILED, 16>(K_GEMM2_TILED, m2, prm, s);
}

// ------------------------------------------------------------ vocab head
struct LmWs {
    int32_t* status;
    __nv_bfloat16* x_pad;
    float* partials;
    size_t bytes;
};

static LmWs lm_ws_layout(void* base, int H, int V) {
    LmWs w{};
    char* p = static_cast<char*>(base);
    size_t off = 0;
    auto take = [&](size_t bytes) -> char* {
        char* r = p ? p + off : nullptr;
        off += align_up(bytes, 1024);
        return r;
    };
    w.status = reinterpret_cast<int32_t*>(take(256));
    w.x_pad = reinterpret_cast<__nv_bfloat16*>(take(static_cast<size_t>(BM) * H * 2));
    w.partials = reinterpret_cast<float*>(take(static_cast<size_t>(BM) * 128 * sizeof(float) * 2 * num_sms()));
    w.bytes = off;
    return w;
}

size_t lm_ws_bytes(int H, int V) { return lm_ws_layout(nullptr, H, V).bytes; }

// keys != nullptr: fused argmax -- no logits; keys [T][V/16] receives the
// per-16-row-chunk argmax keys of every row (see argmax_chunk_store).
ms_status lm_launch(const void* x, const void* wlm, int T, int H, int V, void* logits, void* ws,
                    cudaStream_t s, unsigned long long* keys = nullptr, int32_t* status = nullptr) {
    LmWs w = lm_ws_layout(ws, H, V);
    if (status) w.status = status;
    for (int t0 = 0; t0 < T; t0 += BM) {
        const int tc = T - t0 < BM ? T - t0 : BM;
        const __nv_bfloat16* xc = reinterpret_cast<const __nv_bfloat16*>(x) + static_cast<size_t>(t0) * H;
        ms_status st = launch(K_FFN_PREP, ffn_prep_kernel, dim3(2 * num_sms()), dim3(256), 0, s, xc,
                              static_cast<const int32_t*>(nullptr), tc, H, 0, 0,
                              static_cast<__nv_bfloat16*>(nullptr), w.x_pad, BM, w.status);
        if (st != MS_OK) return st;
        Maps m{};
        bool ok = make_packed_map(&m.w_a, wlm, V, H, 1) && make_packed_map(&m.w_s, wlm, V, H, 1) &&
                  make_map(&m.tok_r, w.x_pad, H, BM, 1, TOKBOX) && make_map(&m.tok_s, w.x_pad, H, BM, 1, TOKBOX);
        if (!ok) return MS_ERR_CUDA;
        Params prm{};
        prm.T = tc; prm.H = H; prm.E = 1; prm.I = BM; prm.S = 0; prm.k = 1; prm.V = V;
        prm.bn = 128;
        prm.offsets = nullptr;
        prm.logits = keys ? nullptr : reinterpret_cast<__nv_bfloat16*>(logits) + static_cast<size_t>(t0) * V;
        prm.amax_key = keys ? keys + static_cast<size_t>(t0) * (V / 16) : nullptr;
        prm.partials = w.partials;
        prm.status = w.status;
        prm.wait_limit_ns = wait_limit_ns();
        prm.dtrace = g_dtrace;
        // the fused argmax: token-major form (all 128 token rows) above 32 tokens,
        // vocabulary-major with warp maxima below
        st = launch_stream<LM_STREAM>(K_LM_HEAD, keys && tc > 32 ? BM : stream_nmax(tc), m, prm, s);
        if (st != MS_OK) return st;
    }
    return MS_OK;
}

// ------------------------------------------------------------ router on the tensor cores
// W_r (fp32) as three bf16 parts hi + mid + lo: hi = bf16(w), mid = bf16(w - hi),
// lo = bf16(w - hi - mid) -- each difference is exact in fp32, and the three
// parts carry the 24-bit significand.  Rows [s][E][H], s = 0, 1, 2.
__global__ void __launch_bounds__(256) route_split_kernel(const float* __restrict__ wr, int n,
                                                          __nv_bfloat16* __restrict__ w3) {
    grid_dep_wait();
    grid_dep_launch();
    for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
        const float w = __ldg(wr + i);
        const __nv_bfloat16 hi = __float2bfloat16_rn(w);
        const float r1 = w - __bfloat162float(hi);
        const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
        const float r2 = r1 - __bfloat162float(mid);
        w3[i] = hi;
        w3[n + i] = mid;
        w3[2 * n + i] = __float2bfloat16_rn(r2);
    }
}

size_t route_tc_ws_bytes(int E, int H) { return align_up(256, 1024) + align_up(static_cast<size_t>(3) * E * H * 2, 1024); }

bool route_tc_supported(int E, int k, int H) {
    return E % 16 == 0 && E <= ROUTE_TC_EMAX && k <= ROUTE_TC_KMAX && H % BK == 0;
}

// logits = xhat [T][H] (bf16) . W_r^T as (xhat . hi^T + xhat . mid^T) + xhat . lo^T
// with exact bf16 products and fp32 accumulation on the tensor cores, 128
// tokens per tile (tiles dealt round-robin to one CTA per SM); softmax and
// top-k in the epilogue.  ws: status word + the split weights.
ms_status route_tc_launch(const void* x, const float* wr, const float* bias, int T, int H, int E, int k, int renorm,
                          int32_t* idx, float* w, void* ws, int32_t* status, cudaStream_t s) {
    char* base = static_cast<char*>(ws);
    auto* w3 = reinterpret_cast<__nv_bfloat16*>(base + align_up(256, 1024));
    const int n = E * H;
    ms_status st = launch(K_ROUTE_SPLIT, route_split_kernel, dim3(std::min((n + 255) / 256, 2 * num_sms())),
                          dim3(256), 0, s, wr, n, w3);
    if (st != MS_OK) return st;
    Maps m{};
    if (!make_map(&m.w_a, w3, H, 3 * E, 1, 3 * E) || !make_map(&m.tok_r, x, H, T, 1, BM)) return MS_ERR_CUDA;
    m.w_s = m.w_a;
    m.tok_s = m.tok_r;
    Params prm{};
    prm.T = T; prm.H = H; prm.E = E; prm.I = BM; prm.S = 0; prm.k = k; prm.V = 0;
    prm.bn = 3 * E;
    prm.offsets = nullptr;
    prm.rbias = bias;
    prm.ridx = idx;
    prm.rw = w;
    prm.rrenorm = renorm;
    prm.nct = num_sms();
    prm.status = status ? status : reinterpret_cast<int32_t*>(base);
    prm.wait_limit_ns = wait_limit_ns();
    prm.dtrace = g_dtrace;
    return launch_gemm<ROUTE_TILED, 16>(K_ROUTE_TC, m, prm, s);
}

// ------------------------------------------------------------ linear layer
// y [T][N] fp32 = x [T][K] . W^T for T <= 128, run as the streaming GEMM2
// schedule with one group (weights are the M operand, the T token rows the N
// operand; split tiles finished by ffn_finish_kernel).  x: bf16 with x_rows
// >= T rows allocated, W: packed [N][K], offsets: device {0, T}.  Scratch:
// linear_ws_bytes(T) for the split-tile partials; status: device word.
size_t linear_ws_bytes(int T) {
    return align_up(static_cast<size_t>(BM) * stream_nmax(T) * 2 * sizeof(float) * 4 * num_sms(), 1024);
}

ms_status linear_launch(const void* x, int x_rows, int T, int K, const void* w, int N, const int32_t* offsets,
                        float* y, void* ws, int32_t* status, cudaStream_t s) {
    if (T > BM || K % 128 != 0 || N % 128 != 0) return MS_ERR_UNSUPPORTED;
    Params prm{};
    prm.T = T; prm.H = N; prm.E = 1; prm.I = K; prm.S = 0; prm.k = 1; prm.V = 0;
    prm.bn = 128;
    prm.offsets = offsets;
    prm.y_perm = y;
    prm.y_bf16 = 0;
    prm.partials = static_cast<float*>(ws);
    prm.status = status;
    prm.wait_limit_ns = wait_limit_ns();
    prm.dtrace = g_dtrace;
    Maps m{};
    if (!make_packed_map(&m.w_a, w, N, K, 1) || !make_map(&m.tok_r, x, K, x_rows, 1, TOKBOX)) return MS_ERR_CUDA;
    m.w_s = m.w_a;
    m.tok_s = m.tok_r;
    return launch_stream<G2_STREAM>(K_GEMM2_STREAM, stream_nmax(T), m, prm, s);
}

}  // namespace ms

extern "C" size_t moe_route_topk_tensor_workspace_size(int E, int H) {
    if (E <= 0 || H <= 0) return 0;
    return ms::route_tc_ws_bytes(E, H);
}

extern "C" ms_status moe_route_topk_tensor(const void* xhat, const float* w_router, const float* logit_bias, int T,
                                           int H, int E, int k, int renormalize, int32_t* topk_idx, float* topk_w,
                                           void* ws, size_t ws_bytes, void* stream) {
    if (!xhat || !w_router || !topk_idx || !topk_w) return MS_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || E <= 0 || k <= 0 || k > E) return MS_ERR_INVALID_ARG;
    if (!ms::route_tc_supported(E, k, H) || H % 128 != 0) return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(xhat) || !ms::aligned16(w_router)) return MS_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ms::route_tc_ws_bytes(E, H)) return MS_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 1023u) return MS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t ce = cudaMemsetAsync(ws, 0, sizeof(int32_t), s);
    if (ce != cudaSuccess) {
        ms::set_cuda_error(ce);
        return MS_ERR_CUDA;
    }
    return ms::route_tc_launch(xhat, w_router, logit_bias, T, H, E, k, renormalize, topk_idx, topk_w, ws, nullptr, s);
}

extern "C" size_t moe_expert_ffn_workspace_size(int T, int H, int E, int I, int S, int k) {
    if (T <= 0 || H <= 0 || E <= 0 || I <= 0 || S < 0 || k <= 0) return 0;
    return ms::ffn_ws_bytes(T, H, E, I, S, k);
}

extern "C" ms_status moe_expert_ffn(const void* xhat, const int32_t* expert_offsets,
                                    const int32_t* perm_token, const void* w_gate_up,
                                    const void* w_down, const void* ws_gate_up,
                                    const void* ws_down, int T, int H, int E, int I, int S, int k,
                                    void* y_perm, ms_dtype y_perm_dtype, float* y_shared, void* ws,
                                    size_t ws_bytes, void* stream) {
    if (!xhat || !expert_offsets || !perm_token || !w_gate_up || !w_down || !y_perm)
        return MS_ERR_INVALID_ARG;
    if (T <= 0 || H <= 0 || E <= 0 || I <= 0 || S < 0 || k <= 0 || k > E) return MS_ERR_INVALID_ARG;
    if (y_perm_dtype != MS_F32 && y_perm_dtype != MS_BF16) return MS_ERR_INVALID_ARG;
    if (S > 0 && (!ws_gate_up || !ws_down || !y_shared)) return MS_ERR_INVALID_ARG;
    if (E > ms::MAX_GROUPS - 1 || H % 128 != 0 || I % 128 != 0 || S > 8) return MS_ERR_UNSUPPORTED;
    if (static_cast<long>(T) * k > (1L << 30)) return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(xhat) || !ms::aligned16(w_gate_up) || !ms::aligned16(w_down) || !ms::aligned16(y_perm) ||
        (S > 0 && (!ms::aligned16(ws_gate_up) || !ms::aligned16(ws_down) || !ms::aligned16(y_shared))))
        return MS_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ms::ffn_ws_bytes(T, H, E, I, S, k)) return MS_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 1023u) return MS_ERR_INVALID_ARG;
    // the status word at ws + 0 reports this call's device-side conditions only
    cudaError_t ce = cudaMemsetAsync(ws, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream));
    if (ce != cudaSuccess) {
        ms::set_cuda_error(ce);
        return MS_ERR_CUDA;
    }
    return ms::ffn_launch(xhat, expert_offsets, perm_token, w_gate_up, w_down, ws_gate_up, ws_down, T, H, E,
                          I, S, k, y_perm, y_perm_dtype, y_shared, ws, static_cast<cudaStream_t>(stream));
}

namespace ms {
ms_status verify_keys_launch(const unsigned long long*, int, int, int, const int32_t*, int32_t*, int32_t*,
                             int32_t*, cudaStream_t);
}

extern "C" size_t spec_verify_lm_head_workspace_size(int B, int K, int H, int V) {
    if (B <= 0 || K < 0 || H <= 0 || V <= 0) return 0;
    return ms::lm_ws_bytes(H, V) + ms::align_up(static_cast<size_t>(B) * (K + 1) * (V / 16) * 8, 1024);
}

extern "C" ms_status spec_verify_lm_head_greedy(const void* xhat, const void* w_lm, const int32_t* draft, int B,
                                                int K, int H, int V, int32_t* argmax, int32_t* committed,
                                                int32_t* n_committed, void* ws, size_t ws_bytes, void* stream) {
    if (!xhat || !w_lm || (K > 0 && !draft) || !argmax || !committed || !n_committed) return MS_ERR_INVALID_ARG;
    if (B <= 0 || K < 0 || H <= 0 || V <= 0) return MS_ERR_INVALID_ARG;
    if (K > 8 || H % 128 != 0 || V % 128 != 0 || V > (1 << 30)) return MS_ERR_UNSUPPORTED;
    if (static_cast<long>(B) * (K + 1) > (1L << 24)) return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(xhat) || !ms::aligned16(w_lm)) return MS_ERR_INVALID_ARG;
    if (!ws || ws_bytes < spec_verify_lm_head_workspace_size(B, K, H, V)) return MS_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 1023u) return MS_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int T = B * (K + 1);
    const size_t lm_bytes = ms::lm_ws_bytes(H, V);
    auto* keys = reinterpret_cast<unsigned long long*>(static_cast<char*>(ws) + lm_bytes);
    // the status word starts at zero; every key slot is written by the head
    cudaError_t ce = cudaMemsetAsync(ws, 0, sizeof(int32_t), s);
    if (ce != cudaSuccess) {
        ms::set_cuda_error(ce);
        return MS_ERR_CUDA;
    }
    ms_status st = ms::lm_launch(xhat, w_lm, T, H, V, nullptr, ws, s, keys);
    if (st != MS_OK) return st;
    return ms::verify_keys_launch(keys, V / 16, B, K, draft, argmax, committed, n_committed, s);
}

extern "C" size_t lm_head_workspace_size(int T, int H, int V) {
    if (T <= 0 || H <= 0 || V <= 0) return 0;
    return ms::lm_ws_bytes(H, V);
}

extern "C" ms_status lm_head_logits(const void* xhat, const void* w_lm, int T, int H, int V,
                                    void* logits_bf16, void* ws, size_t ws_bytes, void* stream) {
    if (!xhat || !w_lm || !logits_bf16 || T <= 0 || H <= 0 || V <= 0) return MS_ERR_INVALID_ARG;
    if (H % 128 != 0 || V % 128 != 0) return MS_ERR_UNSUPPORTED;
    if (!ms::aligned16(xhat) || !ms::aligned16(w_lm) || !ms::aligned16(logits_bf16)) return MS_ERR_INVALID_ARG;
    if (!ws || ws_bytes < ms::lm_ws_bytes(H, V)) return MS_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(ws) & 1023u) return MS_ERR_INVALID_ARG;
    cudaError_t ce = cudaMemsetAsync(ws, 0, sizeof(int32_t), static_cast<cudaStream_t>(stream));
    if (ce != cudaSuccess) {
        ms::set_cuda_error(ce);
        return MS_ERR_CUDA;
    }
    return ms::lm_launch(xhat, w_lm, T, H, V, logits_bf16, ws, static_cast<cudaStream_t>(stream));
}

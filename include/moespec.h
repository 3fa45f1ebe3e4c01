/*
 * moespec -- MoE verify layer and greedy speculative verification for
 * NVIDIA B200 (sm_100a).  C ABI of libmoespec.so.
 *
 * The operation these calls implement is the hot path of the jina-ocr-v1
 * document parser's decoder as its pages describe it:
 *  - a mixture-of-experts decoder layer with 64 routed experts, two shared
 *    experts and top-6 routing (clawpit.io, "Lean architecture with a
 *    compressed encoder"; aikraft.ru, "Архитектура и эффективность"),
 *  - run over the K+1 positions that FastMTP speculative decoding verifies
 *    (K = 3 drafts), followed by greedy verification: accept the longest
 *    prefix of drafts that matches the verifier's own picks and commit one
 *    more token of the verifier's (jina.ai, "Modèle et entraînement";
 *    clawpit.io, "Speculative decoding without accuracy loss").
 * The pages define no programming interface; the calls below follow the
 * steps of that statement.
 *
 * Conventions for every call
 *  - Pointers: every tensor argument is a DEVICE pointer unless stated, in
 *    row-major layout, and must be 16-byte aligned.  bf16 tensors hold IEEE
 *    bfloat16 bit patterns.  The caller owns every buffer; the library never
 *    allocates, frees or retains device memory during a call.
 *  - Scratch: calls that need scratch take (ws, ws_bytes), sized by the
 *    matching *_workspace_size() query; contents need no initialisation and
 *    are clobbered.  ws must not be shared by calls that may overlap.
 *  - Streams: `stream` is a cudaStream_t (NULL = legacy default stream).
 *    Every call is asynchronous on that stream and never synchronises the
 *    host.  Kernels are launched with programmatic dependent launch, so a
 *    call may begin while the previous kernel on the stream drains; each
 *    kernel waits for its predecessor before touching activations, routing
 *    tables, workspace or outputs.  Weights (expert, shared-expert, router
 *    and vocabulary-head weights) are read-only inputs that kernels start
 *    reading before that wait: they must not be written by the work that
 *    immediately precedes the call on its stream.
 *  - Errors: arguments are validated on the host before anything is
 *    launched; a bad argument returns MS_ERR_INVALID_ARG / MS_ERR_UNSUPPORTED
 *    / MS_ERR_WORKSPACE and launches nothing.  A failed launch returns
 *    MS_ERR_CUDA (details via ms_last_cuda_error_string).  Device-side
 *    conditions (a bounded wait that ran out, an out-of-range index seen by
 *    a kernel) are recorded in a status word inside the caller's workspace
 *    and read with ms_device_status(); the kernel then skips the affected
 *    work instead of trapping.
 *  - Sizes: 1 <= k <= E <= 256; H % 128 == 0; I % 128 == 0; 0 <= K <= 8 (K = 0: plain greedy).
 */
#ifndef MOESPEC_H
#define MOESPEC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MS_API __attribute__((visibility("default")))
#else
#define MS_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MS_OK = 0,
    MS_ERR_INVALID_ARG = -1,   /* null pointer, non-positive size, bad enum    */
    MS_ERR_UNSUPPORTED = -2,   /* valid but outside the supported shape set   */
    MS_ERR_WORKSPACE = -3,     /* ws missing or smaller than the size query   */
    MS_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed            */
    MS_ERR_TIMEOUT = -5,       /* a device-side bounded wait ran out           */
    MS_ERR_DEVICE_INDEX = -6,  /* a kernel saw an index outside its range      */
    MS_ERR_DRAIN_TIMEOUT = -7  /* after a timeout, a kernel's wait for its own
                                  in-flight copies/MMAs ran out as well; it
                                  exited without releasing its tensor memory:
                                  the device state is undefined, reset it    */
} ms_status;

typedef enum { MS_F32 = 0, MS_BF16 = 1 } ms_dtype;

/* ---------------------------------------------------------------------- */
/* a0  RMSNorm of the residual stream (the layer's normalised input).
 * xhat_bf16[t,h] = bf16( a[t,h] / sqrt(mean_h(a[t,:]^2) + eps) * gamma[h] )
 * a: [T,H] fp32.  gamma: [H] fp32 or NULL (= 1).  xhat_bf16: [T,H] bf16.
 * The pages do not describe the normalisation; it is the conventional
 * pre-MoE RMSNorm of a DeepSeek-style decoder block. */
MS_API ms_status moe_rmsnorm(const float* a, const float* gamma, int T, int H, float eps,
                      void* xhat_bf16, void* stream);

/* a1  Router: fp32 softmax over E experts and top-k selection
 * (top-6 of 64 routed experts: clawpit.io, "Lean architecture ...").
 * z[t,e] = sum_h xhat[t,h] * w_router[e,h] (+ logit_bias[t,e]), fp32.
 * topk_idx[t,0..k-1]: the k largest z in descending order, equal values
 *   broken towards the lower expert index.
 * topk_w[t,j] = softmax(z[t,:])[topk_idx[t,j]], divided by the sum of the
 *   k selected probabilities when renormalize != 0.
 * xhat: [T,H] bf16.  w_router: [E,H] fp32.  logit_bias: [T,E] fp32 or NULL.
 * topk_idx: [T,k] int32.  topk_w: [T,k] fp32.  No scratch. */
MS_API ms_status moe_route_topk(const void* xhat, const float* w_router, const float* logit_bias,
                         int T, int H, int E, int k, int renormalize,
                         int32_t* topk_idx, float* topk_w, void* stream);

/* a1 on the tensor cores, for prefill-sized batches: the same results as
 * moe_route_topk (same ordering and tie rule; gate weights equal up to fp32
 * rounding) from a tcgen05 GEMM.  W_r is split into three bf16 parts
 * hi + mid + lo that carry its fp32 significand (each part's rounding error is
 * exact in fp32), so xhat . W_r = (xhat . hi + xhat . mid) + xhat . lo with
 * exact bf16 products and fp32 accumulation: the logits agree with the fp32
 * ones to within fp32 rounding of the sums.  Softmax and top-k run in the
 * GEMM's epilogue.  E % 16 == 0, E <= 64, k <= 8, H % 128 == 0.
 * Scratch: moe_route_topk_tensor_workspace_size(E, H) bytes (a status word
 * and the split weights); moe_layer_forward uses this form for T >= 1024. */
MS_API size_t moe_route_topk_tensor_workspace_size(int E, int H);
MS_API ms_status moe_route_topk_tensor(const void* xhat, const float* w_router, const float* logit_bias,
                                       int T, int H, int E, int k, int renormalize,
                                       int32_t* topk_idx, float* topk_w, void* ws, size_t ws_bytes,
                                       void* stream);

/* a2  Permutation: group the T*k (token, slot) pairs by expert, ordered by
 * (expert, token) -- a stable counting sort, bit-exact and deterministic.
 * expert_offsets: [E+1] int32, expert e owns rows [off[e], off[e+1]).
 * perm_token: [T*k] int32, token of each grouped row.
 * slot_of: [T,k] int32, grouped row of pair (t,j).
 * Scratch: moe_permute_workspace_size(T,k,E) bytes (0 is returned, and ws
 * may be NULL, when T*k <= 4096).  Out-of-range expert ids are skipped and
 * flagged (MS_ERR_DEVICE_INDEX) when ws is given. */
MS_API size_t moe_permute_workspace_size(int T, int k, int E);
MS_API ms_status moe_permute(const int32_t* topk_idx, int T, int k, int E,
                      int32_t* expert_offsets, int32_t* perm_token, int32_t* slot_of,
                      void* ws, size_t ws_bytes, void* stream);

/* Weight layout for the tensor-core GEMMs.  A bf16 matrix stack W[n][rows][cols]
 * (cols = the contraction dimension) is repacked once, at load time, into
 * P[n][rows/128][cols/64][128][64]: each 128-row x 64-column tile the GEMMs
 * load is one contiguous 16 KB block, so weight streaming reads whole DRAM
 * pages.  Values are unchanged.  rows % 128 == 0, cols % 64 == 0; w and packed
 * are distinct device buffers of n*rows*cols bf16 each.  The pages do not
 * describe storage; this is the library's own format. */
MS_API ms_status moe_pack_weights(const void* w, int n, int rows, int cols, void* packed, void* stream);

/* a3  Expert FFN: every routed row and the shared experts, SwiGLU.
 * The experts are the decoder's 64 routed and two shared experts (clawpit.io,
 * "Lean architecture with a compressed encoder"; aikraft.ru, "Архитектура и
 * эффективность": 64 routed experts); the pages do not describe an expert's
 * inside, and SwiGLU is the conventional DeepSeek-MoE expert.
 * All four weight arguments are in the packed layout of moe_pack_weights
 * (w_gate_up: n=E, rows=2I, cols=H; w_down: n=E, rows=H, cols=I; shared: n=S).
 * For grouped row r of expert e (token t = perm_token[r]):
 *   g = W_g[e] x_t, u = W_u[e] x_t, h = silu(g) * u (rounded to bf16),
 *   y_perm[r,:] = W_d[e] h            (fp32 accumulation throughout)
 * y_shared[t,:] = sum_s W_d^s (silu(W_g^s x_t) * (W_u^s x_t)).
 * xhat: [T,H] bf16.  w_gate_up: [E,2I,H] bf16 (rows 0..I-1 gate, I..2I-1
 * up).  w_down: [E,H,I] bf16.  ws_gate_up: [S,2I,H] bf16, ws_down: [S,H,I]
 * bf16 (both NULL iff S == 0).  y_perm: [T*k,H] of y_perm_dtype.
 * y_shared: [T,H] fp32 (may be NULL iff S == 0).
 * Tensor-core grouped GEMMs (tcgen05 + TMEM, TMA-fed).  T <= 128 uses a
 * weight-streaming schedule balanced over all SMs; larger T a tiled one.
 * expert_offsets must describe groups inside [0, T*k) of at most T rows
 * each (a token reaches an expert at most once); a group that does not is
 * skipped and flagged MS_ERR_DEVICE_INDEX in the status word, and so is a
 * perm_token entry outside [0, T) (that row's output is then undefined).
 * For T > 128 the token rows are staged through shared memory whole:
 * H <= 12288 there (larger H returns MS_ERR_UNSUPPORTED).
 * Weights in the plain [E,2I,H] / [E,H,I] row-major layout (not passed
 * through moe_pack_weights) are NOT detected: both layouts hold the same
 * number of bf16 values, and the call then returns MS_OK with wrong results.
 * Scratch: moe_expert_ffn_workspace_size(...) bytes; the status word of
 * the bounded waits lives at its start (see ms_device_status). */
MS_API size_t moe_expert_ffn_workspace_size(int T, int H, int E, int I, int S, int k);
MS_API ms_status moe_expert_ffn(const void* xhat, const int32_t* expert_offsets, const int32_t* perm_token,
                         const void* w_gate_up, const void* w_down,
                         const void* ws_gate_up, const void* ws_down,
                         int T, int H, int E, int I, int S, int k,
                         void* y_perm, ms_dtype y_perm_dtype, float* y_shared,
                         void* ws, size_t ws_bytes, void* stream);

/* a4  Combine: gate-weighted un-permute plus residual.
 * Each token's output is the weighted sum of its top-k routed experts plus
 * the two shared experts (clawpit.io, "Lean architecture with a compressed
 * encoder": 64 routed experts, two shared experts, top-6 routing); the
 * shared experts enter with weight 1 and the residual stream is added, the
 * conventional DeepSeek-MoE block (the pages give no formula).
 * out[t,:] = sum_{j<k} topk_w[t,j] * y_perm[slot_of[t,j],:] + y_shared[t,:]
 *            + residual[t,:]            (fp32, in that order)
 * y_perm: [T*k,H] fp32 or bf16.  y_shared, residual: [T,H] fp32 or NULL.
 * out: [T,H] fp32.  out_bf16: [T,H] bf16 copy or NULL.  No scratch. */
MS_API ms_status moe_combine(const void* y_perm, ms_dtype y_perm_dtype, const float* y_shared,
                      const int32_t* slot_of, const float* topk_w, const float* residual,
                      int T, int H, int k, float* out, void* out_bf16, void* stream);

/* a5  Vocab head for the verify rows: logits[t,v] = sum_h xhat[t,h] w_lm[v,h].
 * xhat: [T,H] bf16, w_lm: [V,H] bf16 packed by moe_pack_weights (n=1, rows=V,
 * cols=H), logits: [T,V] bf16 (fp32 accumulate).
 * V % 128 == 0.  Tensor-core GEMM; T is processed 128 rows at a time.
 * Scratch: lm_head_workspace_size(T,H,V) bytes. */
MS_API size_t lm_head_workspace_size(int T, int H, int V);
MS_API ms_status lm_head_logits(const void* xhat, const void* w_lm, int T, int H, int V,
                         void* logits_bf16, void* ws, size_t ws_bytes, void* stream);

/* a6  Greedy verification of one speculative step for B sequences
 * (jina.ai, "Modèle et entraînement"; clawpit.io, "Speculative decoding
 * without accuracy loss"; tau counts the bonus token: jina.ai, "Décodage
 * spéculatif sur un L4").
 * logits: [B,K+1,V] of logits_dtype; row j scores the token after position j
 *   (position 0 = last committed token, 1..K = the drafts).
 * draft: [B,K] int32.
 * argmax[b,j] = argmax_v logits[b,j,v], lowest index among equal maxima;
 * n = longest m <= K with draft[b,i] == argmax[b,i] for all i < m;
 * committed[b,:] = draft[b,0..n-1], argmax[b,n], then -1 padding;
 * n_committed[b] = n + 1, always in 1..K+1.
 * K = 0 (no drafts; draft may be NULL) is plain greedy decoding: one row per
 * sequence, committed[b,0] = its argmax, n_committed[b] = 1.
 * argmax, committed: [B,K+1] int32.  n_committed: [B] int32.
 * Scratch: spec_verify_workspace_size(B,K,V) bytes (partial maxima). */
MS_API size_t spec_verify_workspace_size(int B, int K, int V);
MS_API ms_status spec_verify_greedy(const void* logits, ms_dtype logits_dtype, const int32_t* draft,
                             int B, int K, int V, int32_t* argmax, int32_t* committed,
                             int32_t* n_committed, void* ws, size_t ws_bytes, void* stream);

/* a5 + a6 fused: the vocab head with the verification's argmax in its
 * epilogue, then the prefix match -- the logits are never written.
 * xhat: [B*(K+1),H] bf16, the final hidden states of the verify rows (row
 * b*(K+1)+j scores the token after position j of sequence b).
 * w_lm: [V,H] bf16 packed by moe_pack_weights (n=1, rows=V, cols=H).
 * The argmax of row t is taken over the bf16 rounding of the fp32 logits
 * sum_h xhat[t,h] w_lm[v,h], lowest index among equal values (-0 equals +0),
 * i.e. over exactly the logits lm_head_logits writes; argmax, committed and
 * n_committed then follow spec_verify_greedy (K = 0 included).  K <= 8, H % 128 == 0,
 * V % 128 == 0.  NaN logits are not supported.  Each 16-row vocabulary
 * chunk stores every row's maximum as a 64-bit key (value order << 32 |
 * ~index) in its own slot, and the verify kernel takes each row's largest
 * key: exact, no atomics, deterministic.
 * Scratch: spec_verify_lm_head_workspace_size(B,K,H,V) bytes. */
MS_API size_t spec_verify_lm_head_workspace_size(int B, int K, int H, int V);
MS_API ms_status spec_verify_lm_head_greedy(const void* xhat, const void* w_lm, const int32_t* draft, int B,
                                            int K, int H, int V, int32_t* argmax, int32_t* committed,
                                            int32_t* n_committed, void* ws, size_t ws_bytes, void* stream);

/* FastMTP draft block on the device (jina.ai, "Modèle et entraînement": one
 * dense draft block applied recursively for K prediction steps, shared
 * weights, recursive hidden-state feedback).  The pages leave the block's
 * inside open; this is the multi-token-prediction module without attention:
 *   x  = [bf16(RMSNorm(h)); bf16(RMSNorm(emb[t]))],  u = W_proj x,
 *   h' = u + SwiGLU(bf16(RMSNorm(u))),
 *   t' = argmax bf16(W_lm bf16(RMSNorm(h')))   (lowest index on ties),
 * starting from the verifier's last hidden state h0 and last committed
 * token tok0, each step feeding (h', t') into the next; drafts[b,i] = t' of
 * step i.  RMSNorm: eps 1e-6, no gain.
 * h0: [B,H] fp32.  tok0: [B] int32.  emb: [V,H] bf16 row-major (not packed).
 * w_proj: [H,2H], w_gate_up: [2I,H] (gate rows, then up rows), w_down: [H,I],
 * w_lm: [V,H], all bf16 packed by moe_pack_weights (n = 1).
 * drafts: [B,K] int32.  h_out: [B,H] fp32, the last hidden state, or NULL;
 * distinct from h0.  B <= 128, 1 <= K <= 8, H, I, V multiples of 128.  A
 * token outside [0, V) is flagged MS_ERR_DEVICE_INDEX in the status word at
 * ws + 0 and its embedding taken as zero.
 * Scratch: fastmtp_draft_workspace_size(B,H,I,V) bytes. */
MS_API size_t fastmtp_draft_workspace_size(int B, int H, int I, int V);
MS_API ms_status fastmtp_draft(const float* h0, const int32_t* tok0, const void* emb, const void* w_proj,
                               const void* w_gate_up, const void* w_down, const void* w_lm, int B, int H, int I,
                               int V, int K, int32_t* drafts, float* h_out, void* ws, size_t ws_bytes,
                               void* stream);

/* Allocation-free variant of spec_verify_greedy.  The pages have no
 * counterpart: this exists for callers that cannot allocate device memory,
 * e.g. a plugin running inside an inference server whose device memory is
 * owned by the host application's pool, or a real-time decode loop that must
 * not call cudaMalloc (which may synchronise the device) once it is running.
 * Same arguments and results as spec_verify_greedy, minus (ws, ws_bytes):
 * the partial maxima go to a static 128 KB device array inside the library,
 * which every GPU that loads the library keeps until the process exits.
 * Limit: batches whose partial maxima fit that array -- on a 148-SM B200 any
 * batch with B*(K+1) <= 16384 rows; larger batches return MS_ERR_UNSUPPORTED
 * and launch nothing.  The first call on each device looks the array's device
 * address up (cudaGetSymbolAddress) and caches it; make that first call before
 * any stream capture.  Every call uses the same array, so calls that may
 * overlap on the GPU (other streams, other threads) race and must be ordered
 * by the caller; nothing in it needs to start at zero.  Allocates nothing. */
MS_API ms_status spec_verify_greedy_noalloc(const void* logits, ms_dtype logits_dtype,
                                            const int32_t* draft, int B, int K, int V,
                                            int32_t* argmax, int32_t* committed,
                                            int32_t* n_committed, void* stream);

/* ---------------------------------------------------------------------- */
/* Whole layer in hot-path order: rmsnorm -> route -> permute -> expert FFN
 * -> combine.  a: [T,H] fp32 residual input, out: [T,H] fp32.  Expert weights
 * as for moe_expert_ffn (packed).  The intermediates live in ws
 * (moe_layer_workspace_size bytes).  Results match the five calls made one
 * by one within the layer's tolerance (the fp32 summation order differs
 * between the paths); how they are computed depends on T: up to 16 tokens the
 * whole layer is one persistent kernel (unless batch-invariant schedules are
 * set), up to 128 a chain of the weight-streaming kernels, and from 1,024
 * tokens the router runs on the tensor cores as moe_route_topk_tensor does.
 * Weights must not be written by the work just before the call (see the
 * stream rule above). */
MS_API size_t moe_layer_workspace_size(int T, int H, int E, int I, int S, int k);
MS_API ms_status moe_layer_forward(const float* a, const float* w_router, const float* logit_bias,
                            const void* w_gate_up, const void* w_down,
                            const void* ws_gate_up, const void* ws_down,
                            int T, int H, int E, int I, int S, int k, int renormalize,
                            float* out, void* ws, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------- */
/* Device status word kept at the start of a workspace given to
 * moe_expert_ffn, lm_head_logits or moe_layer_forward.  Each of those calls
 * clears it (stream-ordered) before its first kernel, so it holds the first
 * device-side condition of the most recent call on that workspace.  This
 * synchronises `stream`, returns the word (MS_OK if nothing was recorded)
 * and clears it. */
MS_API ms_status ms_device_status(void* ws, void* stream);

/* Batch-invariant schedules (default off).  The pages call speculative
 * greedy decoding lossless: the tokens it commits are byte-identical to plain
 * greedy decoding (the d9249 blog, "핵심 아이디어 / 구조 / 동작 방식";
 * clawpit.io, "Speculative decoding without accuracy loss").  That holds
 * exactly only if a position's logits do not depend on how many other
 * positions share its forward pass -- K+1 verify rows versus one greedy row.
 * By default the weight-streaming GEMMs (moe_expert_ffn and the layer at
 * T <= 128, lm_head_logits, spec_verify_lm_head_greedy, fastmtp_draft) split
 * output tiles between CTAs at points that depend on the batch, so the last
 * bit of a sum may change with it.  With this setting on, every call issued
 * afterwards (process-wide) computes each output tile whole in one CTA with
 * k in natural order, and moe_layer_forward does not use its fused
 * small-batch kernel: every token's results are then bit-identical whatever
 * else is in the batch (the routing, normalisation, combine and verify are
 * per-token already).  Cost: the tiles are dealt round-robin, without the
 * split that balances them over the SMs.  The prefill-sized (T > 128) tiled
 * path computes each token row whole in any case, in an order of its own. */
MS_API void ms_set_batch_invariant(int on);
MS_API int ms_get_batch_invariant(void);

/* Bounded-wait limit used by every device-side spin (default 1e9 ns). */
MS_API void ms_set_wait_limit_ns(uint64_t ns);
MS_API uint64_t ms_get_wait_limit_ns(void);

/* Self-test of the bounded wait: one kernel spins until *flag == expect or
 * the wait limit passes, then writes MS_OK or MS_ERR_TIMEOUT to *status
 * (device int32).  flag, status: device pointers. */
MS_API ms_status ms_debug_bounded_wait(const int32_t* flag, int32_t expect, int32_t* status,
                                void* stream);

/* In-kernel timeline of the tensor-core GEMMs: while a device buffer of at
 * least 8*256*8 uint64 (128 KB) is set, every CTA of every GEMM launch writes
 * globaltimer stamps (ns) to buf[(row*256 + cta)*8 + slot], row 0..4 =
 * GEMM1 streaming, GEMM2 streaming, vocab head, GEMM1 tiled, GEMM2 tiled;
 * slot 0 entry, 1 schedule built, 2 setup done (after the wait on the previous
 * kernel), 3 first stage of data ready, 4 last MMA issued, 5 epilogue done,
 * 6 loads drained, 7 exit.  Rows 5..7 hold the split-tile finish kernels of
 * the three streaming modes (CTA = blockIdx.x < 256 of the first column
 * chunk): slot 0 entry, 1 after the wait on the GEMM, 3 partials summed, 7
 * exit (only CTAs that finish a tile write slots 3 and 7).  A later launch of the same kind
 * overwrites.  buf = NULL disables it.  For profiling only. */
MS_API ms_status ms_set_device_trace(void* buf, size_t bytes);

/* Launch tracing: when enabled, every kernel this library launches is
 * bracketed by a pair of CUDA events (recorded on the launching stream, so
 * they also work inside stream capture).  ms_trace_read returns, after the
 * stream has completed, the kernel name and duration of entry i. */
MS_API ms_status ms_trace_enable(int capacity);
MS_API void ms_trace_disable(void);
MS_API void ms_trace_reset(void);
MS_API int ms_trace_count(void);
MS_API ms_status ms_trace_read(int i, const char** kernel_name, float* ms);

MS_API const char* ms_status_string(ms_status s);
MS_API const char* ms_last_cuda_error_string(void);
MS_API int ms_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MOESPEC_H */

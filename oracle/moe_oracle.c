/*
 * CPU oracle for the MoE verify layer and the greedy verify step.
 *
 * TEST INFRASTRUCTURE ONLY.  Plain, slow, obviously-correct loops.  Nothing in
 * the product path links, loads or calls this file; only the test-suite, the
 * smoke check and the benchmark's CPU-baseline leg do.  It shares no code,
 * header, table or helper with the CUDA path.
 *
 * Precision: every value is held in fp32 (bf16 inputs are widened exactly);
 * every sum is accumulated in double in a fixed, plain order, so the oracle's
 * own rounding stays far below the tolerances it is used with, and each
 * token's result never depends on which other tokens share the call.
 *
 * Sources (the jina-ocr-v1 pages):
 *  - clawpit.io, "Lean architecture with a compressed encoder": the decoder is
 *    a mixture of experts with 64 routed experts, two shared experts and
 *    top-6 routing.  aikraft.ru, "Архитектура и эффективность": 64 routed
 *    experts.
 *  - jina.ai, "Modèle et entraînement", and clawpit.io, "Speculative decoding
 *    without accuracy loss": the verifier checks the K = 3 drafts greedily,
 *    accepts the longest prefix on which draft and verifier agree, and
 *    commits one token of its own (the bonus when all drafts match), so the
 *    committed text equals plain greedy decoding.
 *  - jina.ai, "Décodage spéculatif sur un L4": tau (tokens committed per
 *    speculative step) counts the bonus token.
 * The pages give neither the gate normalisation nor the expert activation.
 * Readings used here: softmax over all experts then top-k with no
 * renormalisation (a flag turns renormalisation on); SwiGLU experts
 * h = silu(W_g x) * (W_u x), y = W_d h; shared experts added with weight 1;
 * RMSNorm with eps = 1e-6 and unit gain unless a gain vector is given.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define OR_EXPORT __attribute__((visibility("default")))

/* ------------------------------------------------------------- bf16 */

static float or_bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

/* Round to nearest bf16, ties to even (inputs here are finite). */
static uint16_t or_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* Element i of a weight array stored as fp32 (is_bf16 = 0) or bf16 bits. */
static float or_w(const void* w, int is_bf16, size_t i) {
    return is_bf16 ? or_bf16_to_f32(((const uint16_t*)w)[i]) : ((const float*)w)[i];
}

OR_EXPORT void or_f32_to_bf16_array(const float* x, size_t n, uint16_t* out) {
    for (size_t i = 0; i < n; ++i) out[i] = or_f32_to_bf16(x[i]);
}

/* ------------------------------------------------------------- RMSNorm */

/* xhat[t,:] = a[t,:] / sqrt(mean(a[t,:]^2) + eps) * gamma; written as fp32
 * and, rounded to bf16, as the layer's expert input. */
OR_EXPORT void or_rmsnorm(const float* a, const float* gamma, int T, int H, float eps,
                          float* xhat_f32, uint16_t* xhat_bf16) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const float* row = a + (size_t)t * H;
        double ss = 0.0;
        for (int h = 0; h < H; ++h) ss += (double)row[h] * (double)row[h];
        double inv = 1.0 / sqrt(ss / (double)H + (double)eps);
        for (int h = 0; h < H; ++h) {
            double g = gamma ? (double)gamma[h] : 1.0;
            float v = (float)((double)row[h] * inv * g);
            if (xhat_f32) xhat_f32[(size_t)t * H + h] = v;
            if (xhat_bf16) xhat_bf16[(size_t)t * H + h] = or_f32_to_bf16(v);
        }
    }
}

/* ------------------------------------------------------------- router */

/* z[t,e] = sum_h xhat[t,h] * w_router[e,h] (+ bias[t,e]);
 * p[t,:] = softmax(z[t,:]) over all E experts;
 * idx[t,0..k-1] = the k experts with the largest z, in descending z order,
 *                 equal z broken towards the lower expert index;
 * w[t,j] = p[t, idx[t,j]]  (divided by sum_j p[t,idx[t,j]] if renormalize). */
OR_EXPORT void or_route_topk(const float* xhat, const float* w_router, const float* bias,
                             int T, int H, int E, int k, int renormalize,
                             int32_t* idx, float* w, float* logits_out, float* probs_out) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        double* z = (double*)malloc(sizeof(double) * (size_t)E);
        double* p = (double*)malloc(sizeof(double) * (size_t)E);
        char* taken = (char*)calloc((size_t)E, 1);
        for (int e = 0; e < E; ++e) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += (double)xhat[(size_t)t * H + h] * (double)w_router[(size_t)e * H + h];
            /* logits are an fp32 quantity: round once, then add the bias in fp32 */
            float zf = (float)acc;
            if (bias) zf = zf + bias[(size_t)t * E + e];
            z[e] = (double)zf;
            if (logits_out) logits_out[(size_t)t * E + e] = zf;
        }
        double zmax = z[0];
        for (int e = 1; e < E; ++e) if (z[e] > zmax) zmax = z[e];
        double sum = 0.0;
        for (int e = 0; e < E; ++e) { p[e] = exp(z[e] - zmax); sum += p[e]; }
        for (int e = 0; e < E; ++e) {
            p[e] /= sum;
            if (probs_out) probs_out[(size_t)t * E + e] = (float)p[e];
        }
        double wsum = 0.0;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                if (taken[e]) continue;
                if (best < 0 || z[e] > z[best]) best = e;   /* strict: lowest index wins ties */
            }
            taken[best] = 1;
            idx[(size_t)t * k + j] = best;
            wsum += p[best];
        }
        for (int j = 0; j < k; ++j) {
            double pj = p[idx[(size_t)t * k + j]];
            w[(size_t)t * k + j] = (float)(renormalize ? pj / wsum : pj);
        }
        free(z); free(p); free(taken);
    }
}

/* ------------------------------------------------------------- permute */

/* Group the T*k (token, slot) pairs by expert: rows ordered by expert, then by
 * token.  offsets[e] = number of pairs whose expert is < e (offsets[E] = T*k);
 * perm_token[r] = token of row r; slot_of[t,j] = row that holds pair (t,j). */
OR_EXPORT void or_permute(const int32_t* idx, int T, int k, int E,
                          int32_t* offsets, int32_t* perm_token, int32_t* slot_of) {
    for (int e = 0; e <= E; ++e) offsets[e] = 0;
    for (size_t i = 0; i < (size_t)T * k; ++i) offsets[idx[i] + 1] += 1;
    for (int e = 0; e < E; ++e) offsets[e + 1] += offsets[e];
    int32_t* fill = (int32_t*)malloc(sizeof(int32_t) * (size_t)E);
    for (int e = 0; e < E; ++e) fill[e] = offsets[e];
    /* tokens visited in increasing order, so within an expert rows are by token */
    for (int t = 0; t < T; ++t)
        for (int j = 0; j < k; ++j) {
            int e = idx[(size_t)t * k + j];
            int r = fill[e]++;
            perm_token[r] = t;
            slot_of[(size_t)t * k + j] = r;
        }
    free(fill);
}

/* ------------------------------------------------------------- experts */

static double or_silu(double g) { return g / (1.0 + exp(-g)); }

/* One SwiGLU expert applied to one token:
 * g_i = W_gu[i,:] . x, u_i = W_gu[I+i,:] . x, h_i = silu(g_i) * u_i,
 * y[o] = sum_i W_d[o,i] h_i.  w_gu is [2I, H], w_d is [H, I]; y is added
 * into `acc` (double, length H). */
static void or_swiglu_expert(const float* x, const void* w_gu, const void* w_d, int is_bf16,
                             int H, int I, double* h_scratch, double* acc) {
    for (int i = 0; i < I; ++i) {
        double g = 0.0, u = 0.0;
        for (int c = 0; c < H; ++c) {
            g += (double)or_w(w_gu, is_bf16, (size_t)i * H + c) * (double)x[c];
            u += (double)or_w(w_gu, is_bf16, (size_t)(I + i) * H + c) * (double)x[c];
        }
        h_scratch[i] = or_silu(g) * u;
    }
    for (int o = 0; o < H; ++o) {
        double y = 0.0;
        for (int i = 0; i < I; ++i)
            y += (double)or_w(w_d, is_bf16, (size_t)o * I + i) * h_scratch[i];
        acc[o] += y;
    }
}

/* Routed experts: for each selected row r (all T*k rows when rows == NULL),
 * expert e with offsets[e] <= r < offsets[e+1], token t = perm_token[r]:
 * y_perm[r,:] = expert_e(xhat[t,:]).
 * w_gate_up is [E, 2I, H], w_down is [E, H, I] (fp32 or bf16 bits). */
OR_EXPORT void or_expert_ffn_routed(const float* xhat, const void* w_gate_up, const void* w_down,
                                    int is_bf16, const int32_t* offsets, const int32_t* perm_token,
                                    int T, int H, int E, int I, int k,
                                    const int32_t* rows, int n_rows, float* y_perm) {
    (void)T;
    int total = rows ? n_rows : T * k;
#pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < total; ++q) {
        int r = rows ? rows[q] : q;
        int e = 0;
        while (e < E && !(offsets[e] <= r && r < offsets[e + 1])) ++e;
        if (e == E) continue;
        int t = perm_token[r];
        double* hs = (double*)malloc(sizeof(double) * (size_t)I);
        double* acc = (double*)calloc((size_t)H, sizeof(double));
        size_t gu_stride = (size_t)2 * I * H, d_stride = (size_t)H * I;
        const void* gu = is_bf16 ? (const void*)((const uint16_t*)w_gate_up + e * gu_stride)
                                 : (const void*)((const float*)w_gate_up + e * gu_stride);
        const void* dn = is_bf16 ? (const void*)((const uint16_t*)w_down + e * d_stride)
                                 : (const void*)((const float*)w_down + e * d_stride);
        or_swiglu_expert(xhat + (size_t)t * H, gu, dn, is_bf16, H, I, hs, acc);
        for (int o = 0; o < H; ++o) y_perm[(size_t)r * H + o] = (float)acc[o];
        free(hs); free(acc);
    }
}

/* Shared experts: y_shared[t,:] = sum_{s<S} expert_s(xhat[t,:]) for each
 * selected token (all T when tokens == NULL). */
OR_EXPORT void or_expert_ffn_shared(const float* xhat, const void* ws_gate_up, const void* ws_down,
                                    int is_bf16, int T, int H, int I, int S,
                                    const int32_t* tokens, int n_tokens, float* y_shared) {
    int total = tokens ? n_tokens : T;
#pragma omp parallel for schedule(dynamic, 1)
    for (int q = 0; q < total; ++q) {
        int t = tokens ? tokens[q] : q;
        double* hs = (double*)malloc(sizeof(double) * (size_t)I);
        double* acc = (double*)calloc((size_t)H, sizeof(double));
        size_t gu_stride = (size_t)2 * I * H, d_stride = (size_t)H * I;
        for (int s = 0; s < S; ++s) {
            const void* gu = is_bf16 ? (const void*)((const uint16_t*)ws_gate_up + s * gu_stride)
                                     : (const void*)((const float*)ws_gate_up + s * gu_stride);
            const void* dn = is_bf16 ? (const void*)((const uint16_t*)ws_down + s * d_stride)
                                     : (const void*)((const float*)ws_down + s * d_stride);
            or_swiglu_expert(xhat + (size_t)t * H, gu, dn, is_bf16, H, I, hs, acc);
        }
        for (int o = 0; o < H; ++o) y_shared[(size_t)t * H + o] = (float)acc[o];
        free(hs); free(acc);
    }
}

/* ------------------------------------------------------------- combine */

/* out[t,:] = sum_j w[t,j] * y_perm[slot_of[t,j], :] + y_shared[t,:] + residual[t,:] */
OR_EXPORT void or_combine(const float* y_perm, const float* y_shared, const int32_t* slot_of,
                          const float* w, const float* residual, int T, int H, int k,
                          float* out) {
#pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h) {
            double acc = 0.0;
            for (int j = 0; j < k; ++j)
                acc += (double)w[(size_t)t * k + j] *
                       (double)y_perm[(size_t)slot_of[(size_t)t * k + j] * H + h];
            if (y_shared) acc += (double)y_shared[(size_t)t * H + h];
            if (residual) acc += (double)residual[(size_t)t * H + h];
            out[(size_t)t * H + h] = (float)acc;
        }
}

/* ------------------------------------------------------------- vocab head */

/* logits[t,v] = sum_h xhat[t,h] * w_lm[v,h]; w_lm is [V, H]. */
OR_EXPORT void or_lm_head(const float* xhat, const void* w_lm, int is_bf16, int T, int H, int V,
                          float* logits) {
#pragma omp parallel for schedule(static)
    for (int v = 0; v < V; ++v)
        for (int t = 0; t < T; ++t) {
            double acc = 0.0;
            for (int h = 0; h < H; ++h)
                acc += (double)xhat[(size_t)t * H + h] * (double)or_w(w_lm, is_bf16, (size_t)v * H + h);
            logits[(size_t)t * V + v] = (float)acc;
        }
}

/* ------------------------------------------------------------- verify */

/* Greedy verification of one speculative step for each of B sequences.
 * logits is [B, K+1, V]: row j scores the token that follows input position j
 * (position 0 is the last committed token, positions 1..K hold the drafts).
 *   g_j = argmax_v logits[b,j,v], the lowest index among equal maxima;
 *   n   = largest m <= K with draft[b,i] == g_i for every i < m;
 *   committed[b,:] = draft[b,0..n-1], then g_n, then -1 padding;
 *   n_committed[b] = n + 1  (always in 1..K+1; the +1 is the verifier's own
 *   token, the bonus when all K drafts were accepted). */
OR_EXPORT void or_verify_greedy(const float* logits, const int32_t* draft, int B, int K, int V,
                                int32_t* argmax, int32_t* committed, int32_t* n_committed) {
    for (int b = 0; b < B; ++b) {
        for (int j = 0; j <= K; ++j) {
            const float* row = logits + ((size_t)b * (K + 1) + j) * V;
            int best = 0;
            for (int v = 1; v < V; ++v)
                if (row[v] > row[best]) best = v;
            argmax[b * (K + 1) + j] = best;
        }
        int n = 0;
        while (n < K && draft[b * K + n] == argmax[b * (K + 1) + n]) ++n;
        for (int i = 0; i <= K; ++i) committed[b * (K + 1) + i] = -1;
        for (int i = 0; i < n; ++i) committed[b * (K + 1) + i] = draft[b * K + i];
        committed[b * (K + 1) + n] = argmax[b * (K + 1) + n];
        n_committed[b] = n + 1;
    }
}

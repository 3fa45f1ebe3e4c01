"""Pins for the oracle's SwiGLU experts, combine and vocab head.

Special cases reduce to library routines (numpy fp64 matmul with
scipy.special.expit for the one-expert dense MLP), closed forms computed by
hand (tests/golden/swiglu_closed_form.json), and exact identities (two shared
experts = one expert with concatenated intermediates; relabelling experts
changes nothing; zero weights give zero).
"""
import json
import os

import numpy as np
import pytest
import scipy.special

import oracle

pytestmark = pytest.mark.usefixtures("oracle_lib")
GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _dense_swiglu_fp64(x, wgu, wd):
    # y = W_d (silu(W_g x) * (W_u x)) with silu(z) = z * expit(z)
    I = wgu.shape[0] // 2
    g = x.astype(np.float64) @ wgu[:I].astype(np.float64).T
    u = x.astype(np.float64) @ wgu[I:].astype(np.float64).T
    h = g * scipy.special.expit(g) * u
    return h @ wd.astype(np.float64).T


def test_single_expert_is_dense_swiglu_mlp():
    g = np.random.default_rng(10)
    T, H, I = 9, 48, 40
    x = g.standard_normal((T, H)).astype(np.float32)
    wgu = (g.standard_normal((1, 2 * I, H)) * 0.2).astype(np.float32)
    wd = (g.standard_normal((1, H, I)) * 0.2).astype(np.float32)
    idx = np.zeros((T, 1), np.int32)
    off, perm, slot = oracle.permute(idx, 1)
    y = oracle.expert_ffn_routed(x, wgu, wd, off, perm, 1)
    ref = _dense_swiglu_fp64(x, wgu[0], wd[0])
    np.testing.assert_allclose(y[slot[:, 0]], ref, rtol=1e-5, atol=1e-6)


def test_swiglu_closed_form_golden():
    cases = json.load(open(os.path.join(GOLD, "swiglu_closed_form.json")))["cases"]
    for c in cases:
        x = np.array([c["x"]], np.float32)
        wgu = np.array([c["w_gate_up"]], np.float32)
        wd = np.array([c["w_down"]], np.float32)
        off, perm, _ = oracle.permute(np.zeros((1, 1), np.int32), 1)
        y = oracle.expert_ffn_routed(x, wgu, wd, off, perm, 1)
        np.testing.assert_allclose(y[0], c["y"], rtol=1e-6, atol=1e-7, err_msg=c["name"])


def test_zero_weights_give_zero_and_scaling_is_linear_in_w_down():
    g = np.random.default_rng(11)
    T, H, I, E, k = 6, 16, 8, 4, 2
    x = g.standard_normal((T, H)).astype(np.float32)
    wgu = g.standard_normal((E, 2 * I, H)).astype(np.float32)
    wd = g.standard_normal((E, H, I)).astype(np.float32)
    idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    off, perm, _ = oracle.permute(idx, E)
    y0 = oracle.expert_ffn_routed(x, wgu, np.zeros_like(wd), off, perm, k)
    assert np.all(y0 == 0)
    y1 = oracle.expert_ffn_routed(x, wgu, wd, off, perm, k)
    y2 = oracle.expert_ffn_routed(x, wgu, wd * np.float32(2.0), off, perm, k)
    np.testing.assert_array_equal(y2, y1 * np.float32(2.0))


def test_two_shared_equal_one_concatenated():
    g = np.random.default_rng(12)
    T, H, I = 5, 32, 16
    x = g.standard_normal((T, H)).astype(np.float32)
    wgu = (g.standard_normal((2, 2 * I, H)) * 0.3).astype(np.float32)
    wd = (g.standard_normal((2, H, I)) * 0.3).astype(np.float32)
    y2 = oracle.expert_ffn_shared(x, wgu, wd)
    cat_gu = np.concatenate([wgu[0, :I], wgu[1, :I], wgu[0, I:], wgu[1, I:]])[None]
    cat_d = np.concatenate([wd[0], wd[1]], axis=1)[None]
    y1 = oracle.expert_ffn_shared(x, cat_gu, cat_d)
    np.testing.assert_allclose(y2, y1, rtol=1e-6, atol=1e-7)
    ref = _dense_swiglu_fp64(x, wgu[0], wd[0]) + _dense_swiglu_fp64(x, wgu[1], wd[1])
    np.testing.assert_allclose(y2, ref, rtol=1e-5, atol=1e-6)


def test_relabelling_experts_changes_nothing():
    g = np.random.default_rng(13)
    T, H, I, E, k = 7, 16, 8, 5, 2
    x = g.standard_normal((T, H)).astype(np.float32)
    wgu = g.standard_normal((E, 2 * I, H)).astype(np.float32)
    wd = g.standard_normal((E, H, I)).astype(np.float32)
    idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    w = g.random((T, k)).astype(np.float32)
    res = g.standard_normal((T, H)).astype(np.float32)
    off, perm, slot = oracle.permute(idx, E)
    out = oracle.combine(oracle.expert_ffn_routed(x, wgu, wd, off, perm, k), None, slot, w, res)
    pi = g.permutation(E)                      # expert e is stored at pi[e]
    wgu2 = np.empty_like(wgu); wgu2[pi] = wgu
    wd2 = np.empty_like(wd); wd2[pi] = wd
    idx2 = pi[idx].astype(np.int32)
    off2, perm2, slot2 = oracle.permute(idx2, E)
    out2 = oracle.combine(oracle.expert_ffn_routed(x, wgu2, wd2, off2, perm2, k), None, slot2, w, res)
    np.testing.assert_array_equal(out, out2)


def test_bf16_weights_are_widened_exactly():
    g = np.random.default_rng(14)
    T, H, I, E, k = 4, 32, 16, 3, 2
    from speculative_decoding_verification_router_b200 import synth
    x = g.standard_normal((T, H)).astype(np.float32)
    wgu_b = synth.to_bf16_bits(g.standard_normal((E, 2 * I, H)).astype(np.float32))
    wd_b = synth.to_bf16_bits(g.standard_normal((E, H, I)).astype(np.float32))
    idx = np.stack([g.choice(E, k, replace=False) for _ in range(T)]).astype(np.int32)
    off, perm, _ = oracle.permute(idx, E)
    yb = oracle.expert_ffn_routed(x, wgu_b, wd_b, off, perm, k)
    yf = oracle.expert_ffn_routed(x, oracle.widen_bf16(wgu_b), oracle.widen_bf16(wd_b), off, perm, k)
    np.testing.assert_array_equal(yb, yf)


def test_combine_closed_forms():
    g = np.random.default_rng(15)
    T, H, k, S = 6, 10, 3, 2
    res = g.standard_normal((T, H)).astype(np.float32)
    w = g.random((T, k)).astype(np.float32)
    slot = g.permutation(T * k).reshape(T, k).astype(np.int32)
    ones = np.ones((T * k, H), np.float32)
    out = oracle.combine(ones, np.full((T, H), float(S), np.float32), slot, w, res)
    np.testing.assert_allclose(out, res + w.astype(np.float64).sum(1, keepdims=True) + S, rtol=1e-6)
    out0 = oracle.combine(np.zeros((T * k, H), np.float32), None, slot, w, res)
    np.testing.assert_array_equal(out0, res)


def test_combine_is_a_scatter_matrix_product():
    # out = res + P y_perm + y_sh with P[t, slot_of[t,j]] = w[t,j] (numpy matmul)
    g = np.random.default_rng(16)
    T, H, k = 8, 12, 2
    y = g.standard_normal((T * k, H)).astype(np.float32)
    ysh = g.standard_normal((T, H)).astype(np.float32)
    res = g.standard_normal((T, H)).astype(np.float32)
    w = g.random((T, k)).astype(np.float32)
    slot = g.permutation(T * k).reshape(T, k).astype(np.int32)
    P = np.zeros((T, T * k))
    for t in range(T):
        for j in range(k):
            P[t, slot[t, j]] = w[t, j]
    ref = res.astype(np.float64) + P @ y.astype(np.float64) + ysh
    np.testing.assert_allclose(oracle.combine(y, ysh, slot, w, res), ref, rtol=1e-6, atol=1e-6)


def test_lm_head_matches_library_matmul():
    g = np.random.default_rng(17)
    from speculative_decoding_verification_router_b200 import synth
    x = g.standard_normal((5, 64)).astype(np.float32)
    wl = synth.to_bf16_bits((g.standard_normal((300, 64)) * 0.02).astype(np.float32))
    ref = x.astype(np.float64) @ oracle.widen_bf16(wl).astype(np.float64).T
    np.testing.assert_allclose(oracle.lm_head(x, wl), ref, rtol=1e-6, atol=1e-7)


def test_moe_layer_tiny_end_to_end_matches_dense_fp64_restatement():
    # With k = E every expert sees every token; routing order then does not
    # matter and the layer equals res + sum_e p_e expert_e(x) + shared(x).
    g = np.random.default_rng(18)
    from speculative_decoding_verification_router_b200.synth import LayerWeights
    T, H, I, E, S = 4, 32, 8, 4, 1
    lw = LayerWeights((g.standard_normal((E, 2 * I, H)) * 0.2).astype(np.float32),
                      (g.standard_normal((E, H, I)) * 0.2).astype(np.float32),
                      (g.standard_normal((S, 2 * I, H)) * 0.2).astype(np.float32),
                      (g.standard_normal((S, H, I)) * 0.2).astype(np.float32),
                      (g.standard_normal((E, H)) * 0.3).astype(np.float32))
    a = g.standard_normal((T, H)).astype(np.float32)
    r = oracle.moe_layer(a, lw, k=E)
    x = r["xhat"].astype(np.float64)
    p = scipy.special.softmax(x @ lw.w_router.astype(np.float64).T, axis=1)
    ref = a.astype(np.float64) + _dense_swiglu_fp64(x, lw.ws_gate_up[0], lw.ws_down[0])
    for e in range(E):
        ref += p[:, e:e + 1] * _dense_swiglu_fp64(x, lw.w_gate_up[e], lw.w_down[e])
    np.testing.assert_allclose(r["out"], ref, rtol=1e-5, atol=1e-5)

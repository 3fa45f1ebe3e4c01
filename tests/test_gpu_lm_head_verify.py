"""GPU parity of the fused vocab head + greedy verification
(spec_verify_lm_head_greedy): the argmax is taken in the GEMM epilogue over the
bf16-rounded logits, so it must equal, bit for bit, the verification of the
logits lm_head_logits writes -- and the oracle's verification of those same
logits.  Independently of the GPU's rounding, every chosen token's logit is
checked against the oracle's fp64 logits."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ms():
    from speculative_decoding_verification_router_b200 import moespec
    return moespec


def _case(B, K, H, V, seed, w=None):
    T = B * (K + 1)
    x = synth.normal_bf16(seed, f"lmv_x{T}x{H}", (T, H), 1.0)
    if w is None:
        w = synth.normal_bf16(seed, f"lmv_w{V}x{H}", (V, H), 0.02)
    return x, w


def _drafts(am, p, V, seed):
    B, K1 = am.shape
    return synth.drafts(am[:, :K1 - 1], p, V, seed)


def _check_against_unfused(ms, x, w, B, K, seed, p_match=0.6):
    xd, wp = dev(x), ms.pack_weights(dev(w))
    V = w.shape[0]
    logits = ms.lm_head(xd, wp)                                  # [T, V] bf16
    lg = logits.view(B, K + 1, V)
    am0, _, _ = ms.verify_greedy(lg, torch.zeros((B, K), dtype=torch.int32, device="cuda"))
    dr = _drafts(host(am0), p_match, V, seed)
    drd = dev(dr)
    am, cm, n = ms.verify_lm_head_greedy(xd, wp, drd)
    ram, rcm, rn = ms.verify_greedy(lg, drd)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(am), host(ram))
    np.testing.assert_array_equal(host(cm), host(rcm))
    np.testing.assert_array_equal(host(n), host(rn))
    return host(logits), dr, host(am), host(cm), host(n)


SHAPES = [(1, 3, 256, 1024), (4, 3, 256, 2048), (2, 8, 128, 1280), (40, 3, 256, 1152), (8, 1, 256, 128),
          (8, 0, 256, 1024)]


@pytest.mark.parametrize("B,K,H,V", SHAPES, ids=[f"B{b}K{k}H{h}V{v}" for b, k, h, v in SHAPES])
def test_fused_equals_unfused_and_oracle(ms, B, K, H, V):
    x, w = _case(B, K, H, V, seed=3)
    lg, dr, am, cm, n = _check_against_unfused(ms, x, w, B, K, seed=3)
    # the oracle's verification of the very logits the GPU wrote
    oam, ocm, on = oracle.verify_greedy(lg.reshape(B, K + 1, V), dr)
    np.testing.assert_array_equal(am, oam)
    np.testing.assert_array_equal(cm, ocm)
    np.testing.assert_array_equal(n, on)
    # and each chosen token is a maximum of the exact logits within the GPU's rounding:
    # one bf16 rounding of the max (2^-8 relative) plus fp32 accumulation over H terms
    z = oracle.lm_head(oracle.widen_bf16(x), w).astype(np.float64)
    zmax = z.max(axis=1)
    zsel = z[np.arange(z.shape[0]), am.reshape(-1)]
    tol = np.abs(zmax) * 2.0 ** -7 + 1e-5 * np.sqrt(H)
    assert np.all(zmax - zsel <= tol)
    assert set(np.unique(n)).issubset(set(range(1, K + 2)))


def test_fused_full_vocab_batch32(ms):
    # the 12-layer step's head: 32 sequences x 4 rows, V = 129,280, H = 1280
    B, K, H, V = 32, 3, 1280, 129280
    x, w = _case(B, K, H, V, seed=0)
    lg, dr, am, cm, n = _check_against_unfused(ms, x, w, B, K, seed=0, p_match=0.576)
    oam, ocm, on = oracle.verify_greedy(lg.reshape(B, K + 1, V), dr)
    np.testing.assert_array_equal(am, oam)
    np.testing.assert_array_equal(n, on)


def test_fused_ties_go_to_the_lowest_index(ms):
    # vocabulary rows repeat a few patterns, so every row's maximum is shared by
    # many indices, in one tile and across tiles: the lowest index must win
    B, K, H, V = 4, 3, 128, 2048
    base = synth.normal_bf16(5, "lmv_tie_patterns", (7, H), 0.05)
    w = base[np.arange(V) % 7]
    x, _ = _case(B, K, H, V, seed=5, w=w)
    lg, dr, am, cm, n = _check_against_unfused(ms, x, w, B, K, seed=5)
    assert np.all(am < 7)   # the first occurrence of each pattern
    z = oracle.lm_head(oracle.widen_bf16(x), w)
    zb = oracle.widen_bf16(oracle.bf16_round(z))
    ref = np.argmax(zb.reshape(B * (K + 1), V), axis=1)
    # on rows where the oracle's bf16 logits have the same maximal pattern, the index agrees
    same = zb.reshape(-1, V)[np.arange(B * (K + 1)), am.reshape(-1)] == zb.reshape(-1, V).max(axis=1)
    np.testing.assert_array_equal(am.reshape(-1)[same], ref[same])


def test_fused_all_drafts_right_and_first_wrong(ms):
    B, K, H, V = 3, 3, 256, 1024
    x, w = _case(B, K, H, V, seed=9)
    xd, wp = dev(x), ms.pack_weights(dev(w))
    am, _, _ = ms.verify_lm_head_greedy(xd, wp, torch.zeros((B, K), dtype=torch.int32, device="cuda"))
    g = host(am)
    right = dev(np.ascontiguousarray(g[:, :K]))
    _, cm, n = ms.verify_lm_head_greedy(xd, wp, right)
    assert np.all(host(n) == K + 1)
    np.testing.assert_array_equal(host(cm), g)
    wrong = g[:, :K].copy()
    wrong[:, 0] = (wrong[:, 0] + 1) % V
    _, cm, n = ms.verify_lm_head_greedy(xd, wp, dev(wrong))
    assert np.all(host(n) == 1)
    np.testing.assert_array_equal(host(cm)[:, 0], g[:, 0])
    assert np.all(host(cm)[:, 1:] == -1)

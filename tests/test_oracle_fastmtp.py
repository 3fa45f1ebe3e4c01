"""Pins of the oracle's FastMTP draft block (closed forms on special weights,
and the recursion equal to K single steps)."""
import numpy as np

import oracle
from speculative_decoding_verification_router_b200 import synth


def _zero_mlp(H, I):
    return np.zeros((2 * I, H), np.float32), np.zeros((H, I), np.float32)


def test_identity_projection_keeps_the_argmax_of_the_hidden_state():
    # W_proj = [I | 0], no MLP, vocab head = identity (V = H): every step's
    # hidden state is the normalised previous one, so every draft is argmax(h0)
    g = np.random.default_rng(0)
    B, H, I = 6, 32, 16
    h0 = (np.stack([g.permutation(H) for _ in range(B)]) * 0.1 + g.standard_normal((B, H)) * 1e-3).astype(np.float32)
    wp = np.concatenate([np.eye(H), np.zeros((H, H))], axis=1).astype(np.float32)
    wgu, wd = _zero_mlp(H, I)
    emb = synth.to_bf16_bits(g.standard_normal((H, H)).astype(np.float32))
    d, hK = oracle.fastmtp_draft(h0, np.zeros(B, np.int32), emb, wp, wgu, wd, np.eye(H, dtype=np.float32), K=3)
    np.testing.assert_array_equal(d, np.repeat(np.argmax(h0, axis=1)[:, None], 3, axis=1))
    # h_K: K-fold normalisation of h0 (to bf16 each time), which keeps direction and gives rms 1
    np.testing.assert_allclose(np.sqrt((hK ** 2).mean(axis=1)), 1.0, rtol=1e-2)


def test_embedding_projection_follows_the_token_chain():
    # W_proj = [0 | I], no MLP, embeddings one-hot under a permutation pi, vocab
    # head = identity: the draft after token t is pi(t), so the K drafts are
    # pi(tok0), pi(pi(tok0)), ...
    g = np.random.default_rng(1)
    B, H, I, K = 5, 24, 8, 4
    pi = g.permutation(H)
    emb = np.zeros((H, H), np.float32)
    emb[np.arange(H), pi] = 3.0
    wp = np.concatenate([np.zeros((H, H)), np.eye(H)], axis=1).astype(np.float32)
    wgu, wd = _zero_mlp(H, I)
    tok0 = g.integers(0, H, B).astype(np.int32)
    d, _ = oracle.fastmtp_draft(g.standard_normal((B, H)).astype(np.float32), tok0,
                                synth.to_bf16_bits(emb), wp, wgu, wd, np.eye(H, dtype=np.float32), K=K)
    want = np.empty((B, K), np.int32)
    t = tok0
    for i in range(K):
        t = pi[t]
        want[:, i] = t
    np.testing.assert_array_equal(d, want)


def test_recursion_equals_single_steps():
    # K steps in one call = K single-step calls fed with (h, t) of the previous one
    g = np.random.default_rng(2)
    B, H, I, V, K = 4, 64, 32, 96, 3
    bf = lambda shape, std: synth.to_bf16_bits((g.standard_normal(shape) * std).astype(np.float32))
    emb, wp, wgu, wd, wl = bf((V, H), 1.0), bf((H, 2 * H), 0.1), bf((2 * I, H), 0.1), bf((H, I), 0.1), bf((V, H), 0.2)
    h0 = g.standard_normal((B, H)).astype(np.float32)
    t0 = g.integers(0, V, B).astype(np.int32)
    d, hK = oracle.fastmtp_draft(h0, t0, emb, wp, wgu, wd, wl, K=K)
    h, t = h0, t0
    for i in range(K):
        di, h = oracle.fastmtp_draft(h, t, emb, wp, wgu, wd, wl, K=1)
        t = di[:, 0]
        np.testing.assert_array_equal(d[:, i], t)
    np.testing.assert_array_equal(hK, h)


def test_dense_mlp_is_added_to_the_projection():
    # W_proj = [I | 0] makes the projection u = bf16(RMSNorm(h0)) exactly; the
    # block's output is u + MLP(u), and doubling the down projection doubles
    # the MLP's part and nothing else
    g = np.random.default_rng(3)
    B, H, I, V = 4, 32, 16, 40
    bf = lambda shape, std: synth.to_bf16_bits((g.standard_normal(shape) * std).astype(np.float32))
    wp = np.concatenate([np.eye(H), np.zeros((H, H))], axis=1).astype(np.float32)
    wgu = oracle.widen_bf16(bf((2 * I, H), 0.3))
    wd = oracle.widen_bf16(bf((H, I), 0.3))
    emb, wl = bf((V, H), 1.0), bf((V, H), 0.2)
    h0 = g.standard_normal((B, H)).astype(np.float32)
    t0 = g.integers(0, V, B).astype(np.int32)
    u = oracle.widen_bf16(oracle.rmsnorm(h0)[1])
    _, h1 = oracle.fastmtp_draft(h0, t0, emb, wp, wgu, wd, wl, K=1)
    _, h2 = oracle.fastmtp_draft(h0, t0, emb, wp, wgu, 2 * wd, wl, K=1)
    y1, y2 = h1 - u, h2 - u
    assert np.abs(y1).max() > 0.05                       # the MLP contributes
    np.testing.assert_allclose(y2, 2 * y1, rtol=0, atol=4e-6 * np.abs(h2).max())

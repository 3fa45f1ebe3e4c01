"""GPU parity of the FastMTP draft block (fastmtp_draft) against the oracle.

One step from the same (h, t): the hidden state within the layer tolerance
(the GPU rounds the SwiGLU activation to bf16), the draft token equal to the
oracle's unless the oracle's two candidates are within rounding of each other.
K steps on the GPU equal K chained single steps bit for bit, and the
closed-form chain of the special weights (one-hot embeddings under a
permutation) is reproduced exactly."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ms():
    from speculative_decoding_verification_router_b200 import moespec
    return moespec


def _weights(B, H, I, V, seed, lm_std=0.05):
    bf = lambda name, shape, std: synth.normal_bf16(seed, f"mtp_{name}", shape, std)
    return dict(emb=bf("emb", (V, H), 1.0), w_proj=bf("proj", (H, 2 * H), 0.02), w_gu=bf("gu", (2 * I, H), 0.02),
                w_d=bf("d", (H, I), 0.02), w_lm=bf("lm", (V, H), lm_std),
                h0=synth.normal(seed, "mtp_h0", (B, H), 1.0).astype(np.float32),
                tok0=synth.stream(seed, "mtp_tok0").integers(0, V, B).astype(np.int32))


def _gpu(ms, w, h0, tok0, K):
    pk = lambda a: ms.pack_weights(dev(a))
    d, h = ms.fastmtp_draft(dev(h0), dev(tok0), dev(w["emb"]), pk(w["w_proj"]), pk(w["w_gu"][None]),
                            pk(w["w_d"][None]), pk(w["w_lm"]), K)
    torch.cuda.synchronize()
    return host(d), host(h)


def _oracle(w, h0, tok0, K):
    return oracle.fastmtp_draft(h0, tok0, w["emb"], w["w_proj"], w["w_gu"], w["w_d"], w["w_lm"], K)


SHAPES = [(4, 256, 256, 1024), (32, 1280, 7168, 129280)]


@pytest.mark.parametrize("B,H,I,V", SHAPES, ids=[f"B{b}H{h}I{i}V{v}" for b, h, i, v in SHAPES])
def test_fastmtp_step_matches_oracle(ms, B, H, I, V):
    w = _weights(B, H, I, V, seed=0)
    d, h = _gpu(ms, w, w["h0"], w["tok0"], K=1)
    rd, rh = _oracle(w, w["h0"], w["tok0"], K=1)
    assert_close(h, rh, what="h after one draft step")
    # The draft token is the greedy pick of the vocab head on the step's own
    # hidden state: every token must be a maximum of the oracle's logits on the
    # GPU's h (the same head input up to RMSNorm rounding), within the rounding
    # the GPU applies to them -- the same bound as the fused head's test: one
    # bf16 rounding of the maximum (2^-7 relative covers both values' rounding)
    # plus fp32 accumulation over H terms -- and one bf16 ulp (2^-7 relative,
    # taken at the row's largest |x|) of a head input whose fp32 and fp64
    # normalisations round apart, times the largest head weight.
    _, xb = oracle.rmsnorm(h)
    x = oracle.widen_bf16(xb).astype(np.float64)
    z = oracle.lm_head(oracle.widen_bf16(xb), w["w_lm"]).astype(np.float64)
    zmax = z.max(axis=1)
    zsel = z[np.arange(B), d[:, 0]]
    wmax = float(np.abs(oracle.widen_bf16(w["w_lm"])).max())
    tol = np.abs(zmax) * 2.0 ** -7 + 1e-5 * np.sqrt(H) + 2.0 ** -7 * np.abs(x).max(axis=1) * wmax
    assert np.all(zmax - zsel <= tol), np.nonzero(zmax - zsel > tol)[0]
    # and on the oracle's own hidden state the picks agree except where two
    # candidates lie within that bound of each other (a near-tie)
    zr = oracle.lm_head(oracle.widen_bf16(oracle.rmsnorm(rh)[1]), w["w_lm"]).astype(np.float64)
    for b in np.nonzero(d[:, 0] != rd[:, 0])[0]:
        gap = zr[b, rd[b, 0]] - zr[b, d[b, 0]]
        assert gap <= tol[b] + 2 * np.abs(z[b] - zr[b]).max(), (b, gap)


def test_fastmtp_recursion_equals_chained_steps(ms):
    B, H, I, V = 8, 256, 384, 2048
    w = _weights(B, H, I, V, seed=1, lm_std=0.2)
    d3, h3 = _gpu(ms, w, w["h0"], w["tok0"], K=3)
    h, t = w["h0"], w["tok0"]
    for i in range(3):
        di, h = _gpu(ms, w, h, t, K=1)
        t = di[:, 0].copy()
        np.testing.assert_array_equal(d3[:, i], t)
    np.testing.assert_array_equal(h3, h)
    # and the oracle, run the same way, agrees on these well-separated logits
    rd, rh = _oracle(w, w["h0"], w["tok0"], K=3)
    np.testing.assert_array_equal(d3, rd)
    assert_close(h3, rh, what="h after three draft steps")


def test_fastmtp_embedding_chain_closed_form(ms):
    # W_proj = [0 | I], no MLP, one-hot embeddings under a permutation pi,
    # vocab head = identity: the drafts are pi(tok0), pi(pi(tok0)), ...
    B, H, I, K = 16, 256, 128, 5
    V = H
    g = np.random.default_rng(7)
    pi = g.permutation(V)
    emb = np.zeros((V, H), np.float32)
    emb[np.arange(V), pi] = 2.0
    w = dict(emb=synth.to_bf16_bits(emb),
             w_proj=synth.to_bf16_bits(np.concatenate([np.zeros((H, H)), np.eye(H)], axis=1).astype(np.float32)),
             w_gu=np.zeros((2 * I, H), np.uint16), w_d=np.zeros((H, I), np.uint16),
             w_lm=synth.to_bf16_bits(np.eye(H, dtype=np.float32)))
    tok0 = g.integers(0, V, B).astype(np.int32)
    d, _ = _gpu(ms, w, g.standard_normal((B, H)).astype(np.float32), tok0, K)
    want = np.empty((B, K), np.int32)
    t = tok0
    for i in range(K):
        t = pi[t]
        want[:, i] = t
    np.testing.assert_array_equal(d, want)


def test_fastmtp_flags_a_bad_token(ms):
    B, H, I, V = 4, 256, 128, 512
    w = _weights(B, H, I, V, seed=2)
    tok0 = w["tok0"].copy()
    tok0[1] = V + 5
    pk = lambda a: ms.pack_weights(dev(a))
    ws = ms.Workspace(ms.lib().fastmtp_draft_workspace_size(B, H, I, V))
    ms.fastmtp_draft(dev(w["h0"]), dev(tok0), dev(w["emb"]), pk(w["w_proj"]), pk(w["w_gu"][None]),
                     pk(w["w_d"][None]), pk(w["w_lm"]), 2, ws=ws)
    assert ms.device_status(ws) == -6

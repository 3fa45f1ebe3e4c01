"""GPU parity of the two largest configurations at their own size.

* The 12-layer decode step at batch 32, K = 3: 12 x (RMSNorm -> MoE ->
  residual) through moe_layer_forward, then the final RMSNorm, the
  V = 129,280 vocab head and greedy verification (jina.ai, "Modèle et
  entraînement"; clawpit.io, "Lean architecture with a compressed encoder":
  12 decoder layers).  The attention between layers is modelled as an
  N(0, 1) input added to the residual stream, fresh per layer.  Every layer is
  checked on its own: the oracle is fed the GPU's layer input, routing and
  permutation are bit-exact (through the library's routing calls on the same
  input) and the layer output is within the layer tolerance.  The verify
  result is bit-exact against the oracle's verification of the GPU's logits.
  The drift of an independent oracle chain from the GPU chain is reported.
* The 36,992-token prefill layer through moe_layer_forward (the bf16 y_perm
  of the tiled path combined over 221,952 rows), compared on a sample of
  tokens that the oracle recomputes one by one (every token's result depends
  on that token alone).
"""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import assert_close, dev, errs, host
from tests.inputs import GAP, routed_layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ms():
    from speculative_decoding_verification_router_b200 import moespec
    return moespec


def _weights_dev(ms, lw):
    pk = lambda a: ms.pack_weights(dev(a))
    return pk(lw.w_gate_up), pk(lw.w_down), pk(lw.ws_gate_up), pk(lw.ws_down), dev(lw.w_router)


def _clear_gaps(z, k):
    zs = -np.sort(-z.astype(np.float64), axis=1)[:, : k + 1]
    return np.nonzero(np.any(-np.diff(zs, axis=1) <= GAP, axis=1))[0]


def _attention_standin(shp, h, lw, layer, seed=0):
    """a_l ~ N(0, 1) with the rows redrawn until the router's top k+1 logits of
    r = h + a_l are all more than 1e-3 apart (the routing is compared bit for bit)."""
    name = f"step12.attn{layer}"
    a = synth.normal(seed, name, h.shape)
    for attempt in range(20):
        r = (h + a).astype(np.float32)
        _, xb = oracle.rmsnorm(r)
        _, _, z, _ = oracle.route_topk(oracle.widen_bf16(xb), lw.w_router, None, shp.k)
        bad = _clear_gaps(z, shp.k)
        if len(bad) == 0:
            return r
        a = synth.resample_rows(a, bad, seed, attempt, name=name)
    raise RuntimeError("could not draw router inputs with clear gaps")


def test_step12_chain_layer_by_layer_and_verify(ms):
    shp = synth.STEP_B32
    T, H, E, I, S, k, V, B, K = shp.T, shp.H, shp.E, shp.I, shp.S, shp.k, shp.V, shp.B, shp.K
    ws = ms.Workspace(ms.layer_workspace_size(T, H, E, I, S, k))
    h = synth.normal(0, "step12.h0", (T, H))
    h_ref = h.copy()                        # the oracle's own chain, for the drift report
    for layer in range(shp.layers):
        lw = synth.layer_weights(shp, 0, layer)
        r = _attention_standin(shp, h, lw, layer)
        wgu, wd, wsgu, wsd, wr = _weights_dev(ms, lw)
        rd = dev(r)
        out = ms.layer_forward(rd, wr, None, wgu, wd, wsgu, wsd, k, ws=ws)
        assert ms.device_status(ws) == 0, layer
        # the routing of this very input through the library's routing calls
        xh = ms.rmsnorm(rd)
        idx, _ = ms.route_topk(xh, wr, None, k)
        off, perm, slot = ms.permute(idx, E)
        torch.cuda.synchronize()
        ref = oracle.moe_layer(r, lw, k)
        np.testing.assert_array_equal(host(idx), ref["idx"], err_msg=f"layer {layer}")
        np.testing.assert_array_equal(host(off), ref["offsets"], err_msg=f"layer {layer}")
        np.testing.assert_array_equal(host(perm), ref["perm"], err_msg=f"layer {layer}")
        np.testing.assert_array_equal(host(slot), ref["slot"], err_msg=f"layer {layer}")
        o = host(out)
        assert_close(o, ref["out"], what=f"layer {layer} out")
        assert_close(o - r, ref["out"] - r, what=f"layer {layer} moe delta")
        # the independent oracle chain gets the same attention stand-in
        h_ref = oracle.moe_layer((h_ref + (r - h)).astype(np.float32), lw, k)["out"]
        h = o
    # final norm -> vocab head -> greedy verification
    wl = synth.normal_bf16(0, "step12.w_lm", (V, H), shp.weight_std)
    wld = ms.pack_weights(dev(wl))
    xh = ms.rmsnorm(dev(h))
    logits = ms.lm_head(xh, wld)
    torch.cuda.synchronize()
    xb_gpu = ms.bf16_to_bits(xh)
    _, xb_ref = oracle.rmsnorm(h)
    ulps = np.abs(xb_gpu.astype(np.int32) - xb_ref.astype(np.int32))
    assert ulps.max() <= 1 and (ulps == 0).mean() >= 0.99
    lg = host(logits)
    z = oracle.lm_head(oracle.widen_bf16(xb_gpu), wl)
    assert_close(lg, z, max_rel=1e-2, mae=2e-3, what="vocab head logits")
    lgb = ms.bf16_to_bits(logits).reshape(B, K + 1, V)
    am_o, _, _ = oracle.verify_greedy(lgb, np.zeros((B, K), np.int32))
    drafts = synth.drafts(am_o[:, :K], shp.p_match, V, 0)
    am, cm, n = ms.verify_greedy(logits.view(B, K + 1, V), dev(drafts))
    fam, fcm, fn = ms.verify_lm_head_greedy(xh, wld, dev(drafts))
    torch.cuda.synchronize()
    oam, ocm, on = oracle.verify_greedy(lgb, drafts)
    np.testing.assert_array_equal(host(am), oam)
    np.testing.assert_array_equal(host(cm), ocm)
    np.testing.assert_array_equal(host(n), on)
    # the fused head (argmax in the GEMM epilogue) takes the same decisions
    np.testing.assert_array_equal(host(fam), oam)
    np.testing.assert_array_equal(host(fn), on)
    assert set(np.unique(on)).issubset(set(range(1, K + 2)))
    # drift of the GPU chain from the oracle's own 12-layer chain (reported)
    mr, ma = errs(h, h_ref)
    print(f"12-layer drift GPU vs oracle chain: max_rel={mr:.3e} mae={ma:.3e}")
    assert np.isfinite(h).all()


def test_prefill_layer_forward_sampled_tokens(ms):
    shp = synth.PREFILL
    T, H, E, I, S, k = shp.T, shp.H, shp.E, shp.I, shp.S, shp.k
    a, lw, bias = routed_layer_inputs(shp, 0)
    wgu, wd, wsgu, wsd, wr = _weights_dev(ms, lw)
    ws = ms.Workspace(ms.layer_workspace_size(T, H, E, I, S, k))
    out = ms.layer_forward(dev(a), wr, None, wgu, wd, wsgu, wsd, k, ws=ws)
    assert ms.device_status(ws) == 0
    # tokens: a random sample, the first and last, and the tokens at the first
    # and last row of every expert group (tile boundaries of the grouped GEMMs)
    _, xb = oracle.rmsnorm(a)
    idx, _, _, _ = oracle.route_topk(oracle.widen_bf16(xb), lw.w_router, None, k)
    off, perm, _ = oracle.permute(idx, E)
    g = np.random.default_rng(11)
    edge = np.concatenate([perm[off[:-1][np.diff(off) > 0]], perm[off[1:][np.diff(off) > 0] - 1]])
    toks = np.unique(np.concatenate([g.choice(T, 192, replace=False), [0, T - 1], edge]))
    ref = oracle.moe_layer(a[toks], lw, k)
    o = host(out[torch.from_numpy(toks).cuda().long()])
    assert_close(o, ref["out"], what="prefill out (sampled tokens)")
    assert_close(o - a[toks], ref["out"] - a[toks], what="prefill moe delta (sampled tokens)")
    assert torch.isfinite(out).all()

"""A decode step captured as one CUDA graph (CapturedStep) and replayed,
checked against the oracle piece by piece: two MoE layers (B = 1, K = 3: the
layer's single persistent launch), the final RMSNorm, the vocab head and the
greedy verification.  Each piece is fed to the oracle with the graph's own
input to it; routing is compared bit for bit through the layer output's
tolerance and the verification bit for bit on the graph's logits."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import assert_close, dev, host
from tests.inputs import routed_layer_inputs

pytestmark = pytest.mark.gpu


def test_captured_decode_step_matches_oracle():
    from speculative_decoding_verification_router_b200 import moespec as ms
    shp = synth.VERIFY_B1
    T, H, E, I, S, k, B, K = shp.T, shp.H, shp.E, shp.I, shp.S, shp.k, shp.B, shp.K
    V = 4096
    a0, lw0, _ = routed_layer_inputs(shp, 11, layer=0)
    lw1 = synth.layer_weights(shp, 11, 1)
    pk = lambda x: ms.pack_weights(dev(x))
    W = [(dev(lw.w_router), pk(lw.w_gate_up), pk(lw.w_down), pk(lw.ws_gate_up), pk(lw.ws_down)) for lw in (lw0, lw1)]
    w_lm = synth.normal_bf16(11, "cap.wlm", (V, H), 0.02)
    wl = pk(w_lm)
    a_h = torch.from_numpy(a0).pin_memory()
    a_d = torch.empty_like(a_h, device="cuda")
    h = [torch.empty((T, H), dtype=torch.float32, device="cuda") for _ in range(2)]
    xn = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    logits = torch.empty((T, V), dtype=torch.bfloat16, device="cuda")
    draft = torch.zeros((B, K), dtype=torch.int32, device="cuda")
    vout = (torch.empty((B, K + 1), dtype=torch.int32, device="cuda"),
            torch.empty((B, K + 1), dtype=torch.int32, device="cuda"), torch.empty(B, dtype=torch.int32, device="cuda"))
    ws = [ms.Workspace(ms.layer_workspace_size(T, H, E, I, S, k)) for _ in range(2)]
    lmws = ms.Workspace(ms.lib().lm_head_workspace_size(T, H, V))
    vws = ms.Workspace(ms.lib().spec_verify_workspace_size(B, K, V))

    def step():
        a_d.copy_(a_h, non_blocking=True)
        cur = a_d
        for l in range(2):
            ms.layer_forward(cur, W[l][0], None, *W[l][1:], k, ws=ws[l], out=h[l])
            cur = h[l]
        ms.rmsnorm(cur, out=xn)
        ms.lm_head(xn, wl, ws=lmws, out=logits)
        ms.verify_greedy(logits.view(B, K + 1, V), draft, ws=vws, out=vout)

    # drafts that partly match the verifier: from one direct step's argmax
    step()
    torch.cuda.synchronize()
    am0 = host(vout[0])
    d = am0[:, :K].copy()
    d[0, 1] = (d[0, 1] + 1) % V   # the second draft is wrong: 2 committed
    draft.copy_(torch.from_numpy(d.astype(np.int32)))
    captured = ms.CapturedStep(step)
    for t in (h[0], h[1], logits):
        t.zero_()
    captured()
    torch.cuda.synchronize()
    h0, h1 = host(h[0]), host(h[1])
    ref0 = oracle.moe_layer(a0, lw0, k)
    assert_close(h0, ref0["out"], what="layer 0")
    assert_close(h0 - a0, ref0["out"] - a0, what="layer 0 moe delta")
    ref1 = oracle.moe_layer(h0, lw1, k)
    assert_close(h1, ref1["out"], what="layer 1 (oracle fed the graph's layer-0 output)")
    xb = ms.bf16_to_bits(xn)
    _, xb_ref = oracle.rmsnorm(h1)
    assert np.abs(xb.astype(np.int32) - xb_ref.astype(np.int32)).max() <= 1
    lgb = ms.bf16_to_bits(logits)
    assert_close(host(logits), oracle.lm_head(oracle.widen_bf16(xb), w_lm), max_rel=1e-2, mae=2e-3, what="logits")
    oam, ocm, on = oracle.verify_greedy(lgb.reshape(B, K + 1, V), d.astype(np.int32))
    np.testing.assert_array_equal(host(vout[0]), oam)
    np.testing.assert_array_equal(host(vout[1]), ocm)
    np.testing.assert_array_equal(host(vout[2]), on)
    assert int(on[0]) == 2

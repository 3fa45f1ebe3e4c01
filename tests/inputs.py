"""Test-side input preparation on top of the seeded generator.

The router's top-k is compared bit for bit, so the inputs are drawn such that
no token has two of its top k+1 router logits within 1e-3 of each other; the
gaps are measured with the oracle (tests may call it) and offending tokens are
redrawn from fresh substreams.  Drafts are built from the oracle's own argmax.
"""
from __future__ import annotations

import numpy as np

import oracle
from speculative_decoding_verification_router_b200 import synth

GAP = 1e-3


def _bad_rows(z: np.ndarray, k: int) -> np.ndarray:
    zs = -np.sort(-z.astype(np.float64), axis=1)[:, : k + 1]
    return np.nonzero(np.any(-np.diff(zs, axis=1) <= GAP, axis=1))[0]


def routed_layer_inputs(shape: synth.MoEShape, seed: int = 0, layer: int = 0,
                        weight_dtype: str = "bf16", name: str = "residual"):
    """(a [T,H] fp32, LayerWeights, bias or None) with clear router gaps after RMSNorm."""
    lw = synth.layer_weights(shape, seed, layer, weight_dtype)
    bias = synth.router_bias(shape, seed)
    a = synth.normal(seed, f"L{layer}.{name}", (shape.T, shape.H))
    wr = lw.w_router
    for attempt in range(20):
        _, xb = oracle.rmsnorm(a)
        _, _, z, _ = oracle.route_topk(oracle.widen_bf16(xb), wr, bias, shape.k)
        bad = _bad_rows(z, shape.k)
        if len(bad) == 0:
            return a, lw, bias
        a = synth.resample_rows(a, bad, seed, attempt, name=f"L{layer}.{name}")
    raise RuntimeError("could not draw router inputs with clear gaps")


def routed_xhat_inputs(shape: synth.MoEShape, seed: int = 0):
    """(xhat bf16 bits [T,H], w_router, bias) with clear router gaps (router tested alone)."""
    lw = synth.layer_weights(shape, seed)
    bias = synth.router_bias(shape, seed)
    xb = synth.xhat_direct(shape, seed)
    for attempt in range(20):
        _, _, z, _ = oracle.route_topk(oracle.widen_bf16(xb), lw.w_router, bias, shape.k)
        bad = _bad_rows(z, shape.k)
        if len(bad) == 0:
            return xb, lw.w_router, bias
        fresh = synth.normal_bf16(seed, f"xhat.resample{attempt}", (len(bad), shape.H), 1.0)
        xb = xb.copy()
        xb[bad] = fresh
    raise RuntimeError("could not draw router inputs with clear gaps")


def verify_inputs(shape: synth.MoEShape, seed: int = 0, dtype: str = "bf16", V=None):
    """(logits [B,K+1,V], drafts [B,K]) with drafts = oracle argmax w.p. p_match."""
    lg = synth.logits(shape, seed, dtype, V=V)
    am, _, _ = oracle.verify_greedy(lg, np.zeros((shape.B, shape.K), np.int32))
    d = synth.drafts(am[:, : shape.K], shape.p_match, V or shape.V, seed)
    return lg, d

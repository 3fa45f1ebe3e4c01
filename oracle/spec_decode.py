"""Plain greedy vs. speculative greedy decoding on a tiny random decoder.

TEST INFRASTRUCTURE ONLY (part of the oracle).

The pages state the property this file exercises: the verifier checks each
draft greedily and commits the longest prefix on which draft and verifier
agree plus one token of its own, so the committed sequence is the verifier's
own greedy sequence and speculation changes only the time taken (jina.ai,
"Modèle et entraînement"; clawpit.io, "Speculative decoding without accuracy
loss"; the d9249 blog's "핵심 아이디어 / 구조 / 동작 방식" calls the outputs
byte-identical).

The decoder is deliberately small and random: embedding -> L blocks of
[causal prefix-mean mixing -> MoE layer with residual] -> RMSNorm -> vocab
head.  Attention is not part of the pages' hot path; the causal prefix mean
stands in for it so that each position depends on every earlier one.  Every
per-position quantity is computed in a fixed order that does not depend on
how many later positions share the forward pass, which is what makes the
verify pass over K+1 positions reproduce the one-token greedy passes exactly.
"""
from __future__ import annotations

import dataclasses
from typing import List

import numpy as np

from . import moe_layer, rmsnorm, lm_head, widen_bf16, verify_greedy


@dataclasses.dataclass
class TinyDecoder:
    emb: np.ndarray          # [V, H] fp32
    layers: list             # list of objects with LayerWeights fields (fp32)
    w_lm: np.ndarray         # [V, H] fp32
    k: int

    @property
    def V(self) -> int:
        return self.emb.shape[0]


@dataclasses.dataclass
class _LW:
    w_gate_up: np.ndarray
    w_down: np.ndarray
    ws_gate_up: np.ndarray
    ws_down: np.ndarray
    w_router: np.ndarray


def make_decoder(seed: int = 0, V: int = 256, H: int = 64, L: int = 2, E: int = 8, I: int = 64,
                 k: int = 2, S: int = 1) -> TinyDecoder:
    g = np.random.Generator(np.random.PCG64(seed))

    def n(shape, std):
        return (g.standard_normal(shape) * std).astype(np.float32)

    layers = []
    for _ in range(L):
        layers.append(_LW(n((E, 2 * I, H), 0.15), n((E, H, I), 0.15),
                          n((S, 2 * I, H), 0.15), n((S, H, I), 0.15), n((E, H), 0.3)))
    return TinyDecoder(n((V, H), 1.0), layers, n((V, H), 0.5), k)


def perturbed(dec: TinyDecoder, scale: float, seed: int) -> TinyDecoder:
    """A drafter: the verifier's weights plus relative Gaussian noise."""
    g = np.random.Generator(np.random.PCG64(seed + 7919))

    def p(a):
        return (a + scale * np.std(a) * g.standard_normal(a.shape)).astype(np.float32)

    layers = [_LW(p(l.w_gate_up), p(l.w_down), p(l.ws_gate_up), p(l.ws_down), p(l.w_router))
              for l in dec.layers]
    return TinyDecoder(p(dec.emb), layers, p(dec.w_lm), dec.k)


def forward(dec: TinyDecoder, tokens: List[int]) -> np.ndarray:
    """Logits [n, V] for every position of `tokens` (row p scores token p+1)."""
    h = dec.emb[np.asarray(tokens, np.int64)].astype(np.float32)
    n = h.shape[0]
    denom = np.arange(1, n + 1, dtype=np.float32)[:, None]
    for lw in dec.layers:
        prefix_mean = np.cumsum(h, axis=0, dtype=np.float32) / denom
        u = (h + prefix_mean).astype(np.float32)
        h = moe_layer(u, lw, dec.k)["out"]
    _, xb = rmsnorm(h)
    return lm_head(widen_bf16(xb), dec.w_lm)


def greedy_decode(dec: TinyDecoder, prompt: List[int], n_new: int) -> List[int]:
    """Plain greedy decoding: one forward per new token, argmax of the last row."""
    toks = list(prompt)
    out: List[int] = []
    while len(out) < n_new:
        lg = forward(dec, toks)
        nxt = int(np.argmax(lg[-1]))       # first maximal index
        toks.append(nxt)
        out.append(nxt)
    return out


def speculative_decode(verifier: TinyDecoder, drafter, prompt: List[int], n_new: int, K: int):
    """Speculative greedy decoding with K drafts per step.

    `drafter(tokens, K)` returns K proposed tokens given the committed ones.
    Each step runs the verifier once over [last committed, d_1..d_K] (with the
    full prefix as context) and commits what `verify_greedy` accepts.
    Returns (tokens, taus) with taus[i] = tokens committed at step i."""
    toks = list(prompt)
    out: List[int] = []
    taus: List[int] = []
    while len(out) < n_new:
        d = [int(x) for x in drafter(toks, K)]
        lg = forward(verifier, toks + d)
        rows = lg[len(toks) - 1: len(toks) + K]            # K+1 rows
        _, committed, ncom = verify_greedy(rows[None, :, :], np.asarray([d], np.int32))
        c = [int(x) for x in committed[0, : int(ncom[0])]]
        toks += c
        out += c
        taus.append(int(ncom[0]))
    return out[:n_new], taus


def greedy_drafter(dec: TinyDecoder):
    """Drafts K tokens by greedy decoding on `dec` (a perturbed or exact copy)."""
    def draft(toks, K):
        ctx = list(toks)
        d = []
        for _ in range(K):
            nxt = int(np.argmax(forward(dec, ctx)[-1]))
            d.append(nxt)
            ctx.append(nxt)
        return d
    return draft


def wrong_drafter(verifier: TinyDecoder):
    """Proposes a first draft that the verifier never picks: its next token + 1."""
    def draft(toks, K):
        g0 = int(np.argmax(forward(verifier, toks)[-1]))
        return [(g0 + 1) % verifier.V] * K
    return draft

"""Seeded synthetic inputs for the MoE verify layer and the greedy verify step.

This module only draws random numbers and lays them out; it holds none of the
method's arithmetic (no normalisation, routing, expert math, argmax or
acceptance).  Both the CPU oracle and the CUDA path are fed from here, so the
two sides always see bit-identical inputs.

Every tensor comes from its own PCG64 substream, keyed by (seed, name), so a
tensor's values do not depend on which other tensors were drawn first.

Workload shapes follow the jina-ocr-v1 pages (decoder: 12 layers, 64 routed
experts, 2 shared experts, top-6 routing -- clawpit.io "Lean architecture";
FastMTP with K = 3 drafts -- jina.ai "Modele et entrainement", clawpit.io
"Speculative decoding without accuracy loss"; up to 1,156 visual tokens per
page -- nullbot.ai "Encodage visuel").  Hidden size, expert width and vocab
are not on the pages; they are fixed here as workload parameters.
"""
from __future__ import annotations

import dataclasses
import hashlib
from typing import Optional

import numpy as np


# ---------------------------------------------------------------- workloads

@dataclasses.dataclass(frozen=True)
class MoEShape:
    name: str
    B: int          # sequences in the verify batch
    K: int          # drafts per sequence; each sequence contributes K+1 rows
    H: int          # hidden size
    E: int          # routed experts
    I: int          # SwiGLU intermediate width of one expert
    k: int          # experts chosen per token
    S: int          # shared experts (see every token)
    V: int          # vocabulary of the verify head
    router_std: float
    weight_std: float = 0.02
    dirichlet_alpha: Optional[float] = None   # per-sequence expert preference
    tokens: Optional[int] = None              # overrides B*(K+1) (prefill)
    layers: int = 1
    p_match: float = 0.6                      # draft == verifier pick

    @property
    def T(self) -> int:
        return self.tokens if self.tokens is not None else self.B * (self.K + 1)


# Tiny case: 4 sequences x (K+1)=4 positions, hidden 256, 8 experts.
TINY = MoEShape("tiny_t16_h256_e8", B=4, K=3, H=256, E=8, I=128, k=2, S=1,
                V=1024, router_std=0.05, p_match=0.6)
# Batch-1 decode verify layer: 4 tokens, weight-bandwidth bound.
VERIFY_B1 = MoEShape("verify_b1_k3_h1280_e64", B=1, K=3, H=1280, E=64, I=896,
                     k=6, S=2, V=129280, router_std=0.05)
# Concurrency-32 verify layer, skewed expert load.
VERIFY_B32 = MoEShape("verify_b32_k3_h1280_e64_skew", B=32, K=3, H=1280, E=64,
                      I=896, k=6, S=2, V=129280, router_std=0.05,
                      dirichlet_alpha=0.3)
# 12-layer decode step + vocab head + greedy verify, batch 32.
STEP_B32 = MoEShape("step12_b32_k3_v129280", B=32, K=3, H=1280, E=64, I=896,
                    k=6, S=2, V=129280, router_std=0.05, layers=12,
                    p_match=0.576)
# Prefill-sized layer: 32 pages x 1,156 visual tokens.
PREFILL = MoEShape("prefill_t36992_h1280_e64", B=32, K=0, H=1280, E=64, I=896,
                   k=6, S=2, V=129280, router_std=1.0 / np.sqrt(1280.0),
                   tokens=32 * 1156)

WORKLOADS = {w.name: w for w in (TINY, VERIFY_B1, VERIFY_B32, STEP_B32, PREFILL)}


# ---------------------------------------------------------------- streams

def stream(seed: int, name: str) -> np.random.Generator:
    """Independent PCG64 generator for tensor `name` under `seed`."""
    h = int.from_bytes(hashlib.sha256(name.encode()).digest()[:8], "little")
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, h])))


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); uint16 bits.

    Input preparation only: the generated bf16 numbers *are* the inputs."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    r = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal(seed: int, name: str, shape, std: float = 1.0) -> np.ndarray:
    g = stream(seed, name)
    out = g.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        out *= np.float32(std)
    return out


def normal_bf16(seed: int, name: str, shape, std: float) -> np.ndarray:
    return to_bf16_bits(normal(seed, name, shape, std))


# ---------------------------------------------------------------- tensors

@dataclasses.dataclass
class LayerWeights:
    w_gate_up: np.ndarray   # [E, 2I, H] bf16 bits; rows 0..I-1 gate, I..2I-1 up
    w_down: np.ndarray      # [E, H, I] bf16 bits
    ws_gate_up: Optional[np.ndarray]   # [S, 2I, H] bf16 bits
    ws_down: Optional[np.ndarray]      # [S, H, I] bf16 bits
    w_router: np.ndarray    # [E, H] fp32


def layer_weights(shape: MoEShape, seed: int = 0, layer: int = 0,
                  weight_dtype: str = "bf16") -> LayerWeights:
    """Expert and router weights of one MoE layer.

    weight_dtype "bf16" returns bf16 bit patterns (uint16); "f32" returns the
    same draws unrounded (float32), for the fp32 variant of the tiny case."""
    E, I, H, S = shape.E, shape.I, shape.H, shape.S
    pre = f"L{layer}."
    conv = to_bf16_bits if weight_dtype == "bf16" else (lambda a: a)
    wgu = conv(normal(seed, pre + "w_gate_up", (E, 2 * I, H), shape.weight_std))
    wd = conv(normal(seed, pre + "w_down", (E, H, I), shape.weight_std))
    if S > 0:
        wsgu = conv(normal(seed, pre + "ws_gate_up", (S, 2 * I, H), shape.weight_std))
        wsd = conv(normal(seed, pre + "ws_down", (S, H, I), shape.weight_std))
    else:
        wsgu = wsd = None
    wr = normal(seed, pre + "w_router", (E, H), shape.router_std)
    return LayerWeights(wgu, wd, wsgu, wsd, wr)


def residual(shape: MoEShape, seed: int = 0, name: str = "residual") -> np.ndarray:
    """Layer input a ~ N(0, 1), [T, H] fp32 (normalised by the layer itself)."""
    return normal(seed, name, (shape.T, shape.H))


def xhat_direct(shape: MoEShape, seed: int = 0, name: str = "xhat") -> np.ndarray:
    """Unit-variance activations already in bf16, [T, H] bf16 bits.

    Used where a call is tested on its own and its input is the normalised
    activation; an N(0,1) row has RMS close to 1."""
    return normal_bf16(seed, name, (shape.T, shape.H), 1.0)


def router_bias(shape: MoEShape, seed: int = 0, name: str = "router_bias") -> Optional[np.ndarray]:
    """Per-sequence expert preference as an additive logit bias [T, E] fp32.

    Each sequence draws p ~ Dirichlet(alpha * 1_E) and every one of its K+1
    rows gets bias ln(max(p, 1e-6)); None when the workload has no skew."""
    if shape.dirichlet_alpha is None:
        return None
    g = stream(seed, name)
    p = g.dirichlet(np.full(shape.E, shape.dirichlet_alpha), size=shape.B)
    b = np.log(np.maximum(p, 1e-6)).astype(np.float32)
    return np.repeat(b, shape.K + 1, axis=0)


def logits(shape: MoEShape, seed: int = 0, dtype: str = "bf16",
           name: str = "logits", V: Optional[int] = None):
    """Verify-head logits [B, K+1, V] ~ N(0, 1); bf16 bits or float32."""
    V = V or shape.V
    z = normal(seed, name, (shape.B, shape.K + 1, V))
    return to_bf16_bits(z) if dtype == "bf16" else z


def drafts(true_next: np.ndarray, p_match: float, V: int, seed: int = 0,
           name: str = "drafts") -> np.ndarray:
    """Draft tokens [B, K]: the given token w.p. p_match, else uniform in [0, V).

    `true_next[b, i]` is the token the verifier would pick at position i; the
    caller supplies it (this module does not compute it)."""
    g = stream(seed, name)
    B, K = true_next.shape
    keep = g.random((B, K)) < p_match
    rnd = g.integers(0, V, size=(B, K), dtype=np.int64)
    return np.where(keep, true_next, rnd).astype(np.int32)


def resample_rows(x: np.ndarray, rows: np.ndarray, seed: int, attempt: int,
                  name: str = "residual") -> np.ndarray:
    """Replace the given rows of x by fresh N(0,1) draws from a new substream."""
    out = x.copy()
    if len(rows):
        fresh = normal(seed, f"{name}.resample{attempt}", (len(rows), x.shape[1]))
        out[rows] = fresh
    return out

"""Reporting formulas for speculative verification.

Definitions follow the jina-ocr-v1 pages (jina.ai, "Décodage spéculatif sur
un L4"): tau is the mean number of tokens committed per speculative step,
bonus token included; c = tau / S is the cost of one speculative step in units
of one autoregressive step, where S is the measured speedup.  The acceptance
rate the pages quote next to tau (57.6 % at tau = 2.73, K = 3; clawpit.io,
"High throughput on cheap hardware") equals (tau - 1) / K.
"""
from __future__ import annotations


def acceptance_rate(tau: float, K: int) -> float:
    """Fraction of drafts accepted: (tau - 1) / K (the bonus token is not a draft)."""
    return (tau - 1.0) / K


def step_cost(tau: float, speedup: float) -> float:
    """Cost of one speculative step in autoregressive steps: c = tau / S."""
    return tau / speedup


def spec_overhead_s(cost: float, ar_tokens_per_s: float) -> float:
    """Extra time of a speculative step over one autoregressive step, in seconds."""
    return (cost - 1.0) / ar_tokens_per_s


def expected_tau_iid(p: float, K: int) -> float:
    """E[tau] when each draft matches independently with probability p.

    n accepted drafts is the first mismatch position, so P(n >= i) = p**i and
    E[tau] = E[n] + 1 = sum_{i=0..K} p**i."""
    return sum(p ** i for i in range(K + 1))


def verified_tokens_per_s(B: int, K: int, seconds: float) -> float:
    """Rows scored by one verify pass per second: B sequences x (K+1) positions."""
    return B * (K + 1) / seconds

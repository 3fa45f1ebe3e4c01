"""CPU oracle for the MoE verify layer and the greedy verify step.

TEST INFRASTRUCTURE ONLY: imported by the test-suite, by the smoke check and
by the benchmark's CPU-baseline / reference leg, never by the product path.
It shares no code with the CUDA library (the C source is `moe_oracle.c`, built
here with gcc); the only thing both sides share is the seeded input generator.

Every function takes and returns numpy arrays.  bf16 tensors are passed as
uint16 bit patterns and widened exactly inside the C code, so the oracle sees
the very values the GPU sees.

Pinned by the tests in tests/test_oracle_*.py (closed forms, invariants,
brute force on tiny inputs, library routines on special cases, the pages'
printed numbers for the reporting identities).  Every function below has at
least one such pin.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile moe_oracle.c into liboracle.so (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
               "-fvisibility=hidden", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            _lib = ctypes.CDLL(_LIB)
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def _i32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.int32)


def _weights(w):
    """(array, is_bf16) for a weight given as uint16 bf16 bits or float32."""
    if w is None:
        return None, 0
    if w.dtype == np.uint16:
        return np.ascontiguousarray(w), 1
    return np.ascontiguousarray(w, dtype=np.float32), 0


def num_threads() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


# ----------------------------------------------------------------- steps

def rmsnorm(a, gamma=None, eps: float = 1e-6):
    """(xhat fp32 [T,H], xhat bf16 bits [T,H]) = RMSNorm(a)."""
    a = _f32(a)
    T, H = a.shape
    xf = np.empty((T, H), np.float32)
    xb = np.empty((T, H), np.uint16)
    _load().or_rmsnorm(_p(a), _p(_f32(gamma)), ctypes.c_int(T), ctypes.c_int(H),
                       ctypes.c_float(eps), _p(xf), _p(xb))
    return xf, xb


def bf16_round(x):
    """Round fp32 -> bf16 bits (nearest, ties to even), the oracle's own rounding."""
    x = _f32(x)
    out = np.empty(x.shape, np.uint16)
    _load().or_f32_to_bf16_array(_p(x), ctypes.c_size_t(x.size), _p(out))
    return out


def widen_bf16(b):
    """Exact bf16 bits -> fp32."""
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def route_topk(xhat, w_router, bias=None, k: int = 6, renormalize: bool = False):
    """Router: returns (idx [T,k] int32, w [T,k] fp32, logits [T,E], probs [T,E])."""
    xhat = _f32(xhat)
    w_router = _f32(w_router)
    T, H = xhat.shape
    E = w_router.shape[0]
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    z = np.empty((T, E), np.float32)
    p = np.empty((T, E), np.float32)
    _load().or_route_topk(_p(xhat), _p(w_router), _p(_f32(bias)), ctypes.c_int(T), ctypes.c_int(H),
                          ctypes.c_int(E), ctypes.c_int(k), ctypes.c_int(int(renormalize)),
                          _p(idx), _p(w), _p(z), _p(p))
    return idx, w, z, p


def permute(idx, E: int):
    """Group (token, slot) pairs by expert: (offsets [E+1], perm_token [T*k], slot_of [T,k])."""
    idx = _i32(idx)
    T, k = idx.shape
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    slot = np.empty((T, k), np.int32)
    _load().or_permute(_p(idx), ctypes.c_int(T), ctypes.c_int(k), ctypes.c_int(E),
                       _p(offsets), _p(perm), _p(slot))
    return offsets, perm, slot


def expert_ffn_routed(xhat, w_gate_up, w_down, offsets, perm_token, k: int, rows=None):
    """y_perm [T*k, H] (rows not selected are left as NaN)."""
    xhat = _f32(xhat)
    T, H = xhat.shape
    wgu, isb = _weights(w_gate_up)
    wd, isb2 = _weights(w_down)
    assert isb == isb2
    E, twoI, H2 = wgu.shape
    assert H2 == H
    I = twoI // 2
    y = np.full((T * k, H), np.nan, np.float32)
    rows_a = _i32(rows)
    _load().or_expert_ffn_routed(_p(xhat), _p(wgu), _p(wd), ctypes.c_int(isb), _p(_i32(offsets)),
                                 _p(_i32(perm_token)), ctypes.c_int(T), ctypes.c_int(H),
                                 ctypes.c_int(E), ctypes.c_int(I), ctypes.c_int(k),
                                 _p(rows_a), ctypes.c_int(0 if rows_a is None else len(rows_a)),
                                 _p(y))
    return y


def expert_ffn_shared(xhat, ws_gate_up, ws_down, tokens=None):
    """y_shared [T, H] = sum over shared experts (tokens not selected are NaN)."""
    xhat = _f32(xhat)
    T, H = xhat.shape
    wgu, isb = _weights(ws_gate_up)
    wd, _ = _weights(ws_down)
    S, twoI, _ = wgu.shape
    I = twoI // 2
    y = np.full((T, H), np.nan, np.float32)
    tok = _i32(tokens)
    _load().or_expert_ffn_shared(_p(xhat), _p(wgu), _p(wd), ctypes.c_int(isb), ctypes.c_int(T),
                                 ctypes.c_int(H), ctypes.c_int(I), ctypes.c_int(S), _p(tok),
                                 ctypes.c_int(0 if tok is None else len(tok)), _p(y))
    return y


def combine(y_perm, y_shared, slot_of, w, residual):
    """out [T,H] = residual + sum_j w[t,j] y_perm[slot_of[t,j]] + y_shared."""
    y_perm = _f32(y_perm)
    slot_of = _i32(slot_of)
    T, k = slot_of.shape
    H = y_perm.shape[1]
    out = np.empty((T, H), np.float32)
    _load().or_combine(_p(y_perm), _p(_f32(y_shared)), _p(slot_of), _p(_f32(w)), _p(_f32(residual)),
                       ctypes.c_int(T), ctypes.c_int(H), ctypes.c_int(k), _p(out))
    return out


def lm_head(xhat, w_lm):
    """logits [T, V] = xhat @ w_lm^T (w_lm [V, H], bf16 bits or fp32)."""
    xhat = _f32(xhat)
    T, H = xhat.shape
    w, isb = _weights(w_lm)
    V = w.shape[0]
    out = np.empty((T, V), np.float32)
    _load().or_lm_head(_p(xhat), _p(w), ctypes.c_int(isb), ctypes.c_int(T), ctypes.c_int(H),
                       ctypes.c_int(V), _p(out))
    return out


def verify_greedy(logits, draft):
    """Greedy verify: (argmax [B,K+1], committed [B,K+1] (-1 padded), n_committed [B]).

    logits: [B, K+1, V] fp32, or bf16 bits (uint16) which are widened exactly."""
    if logits.dtype == np.uint16:
        logits = widen_bf16(logits)
    logits = _f32(logits)
    draft = _i32(draft)
    B, K1, V = logits.shape
    K = K1 - 1
    assert draft.shape == (B, K)
    am = np.empty((B, K1), np.int32)
    cm = np.empty((B, K1), np.int32)
    n = np.empty(B, np.int32)
    _load().or_verify_greedy(_p(logits), _p(draft), ctypes.c_int(B), ctypes.c_int(K),
                             ctypes.c_int(V), _p(am), _p(cm), _p(n))
    return am, cm, n


# ----------------------------------------------------------------- layer

def moe_layer(a, lw, k: int, bias=None, renormalize: bool = False, eps: float = 1e-6):
    """One MoE layer in the order of the hot path.

    a: residual [T,H] fp32.  lw: synth.LayerWeights.  Returns a dict with every
    intermediate (xhat, idx, w, offsets, perm, slot, y_perm, y_shared, out)."""
    xf, xb = rmsnorm(a, eps=eps)
    x = widen_bf16(xb)          # the experts see the bf16-rounded activation
    idx, w, z, p = route_topk(x, lw.w_router, bias, k, renormalize)
    E = lw.w_router.shape[0]
    off, perm, slot = permute(idx, E)
    y = expert_ffn_routed(x, lw.w_gate_up, lw.w_down, off, perm, k)
    ysh = expert_ffn_shared(x, lw.ws_gate_up, lw.ws_down) if lw.ws_gate_up is not None else None
    out = combine(y, ysh, slot, w, a)
    return dict(xhat_bf16=xb, xhat=x, idx=idx, w=w, logits=z, probs=p, offsets=off, perm=perm,
                slot=slot, y_perm=y, y_shared=ysh, out=out)


def fastmtp_draft(h0, tok0, emb, w_proj, w_gate_up, w_down, w_lm, K: int, eps: float = 1e-6):
    """FastMTP draft block applied recursively for K steps with shared weights
    (jina.ai, "Modèle et entraînement": one dense draft block reused for every
    prediction step, trained with recursive hidden-state feedback; the d9249
    blog's component table: a shared dense draft block, K = 3).

    The pages do not describe the block's inside; this is the multi-token-
    prediction module of the decoder family it extends, without attention:
      x   = [bf16(RMSNorm(h)); bf16(RMSNorm(emb[t]))]        (2H)
      u   = W_proj x                                          (H; W_proj [H, 2H])
      h'  = u + SwiGLU(bf16(RMSNorm(u)))                      (dense, w_gate_up [2I, H], w_down [H, I])
      t'  = argmax_v bf16(W_lm bf16(RMSNorm(h')))_v           (the verifier's vocab head; lowest index on ties)
    starting from the verifier's last hidden state h0 and last committed token
    tok0, each step feeding (h', t') into the next.

    h0 [B,H] fp32, tok0 [B] int32, emb [V,H] bf16 bits, w_proj [H,2H],
    w_gate_up [2I,H], w_down [H,I], w_lm [V,H] (bf16 bits or fp32).
    Returns (drafts [B,K] int32, h_K [B,H] fp32)."""
    h = _f32(h0)
    t = _i32(tok0)
    B, H = h.shape
    emb = np.ascontiguousarray(emb)
    wgu = np.ascontiguousarray(w_gate_up)[None]
    wd = np.ascontiguousarray(w_down)[None]
    rows = np.arange(B, dtype=np.int32)
    drafts = np.empty((B, K), np.int32)
    for i in range(K):
        _, hb = rmsnorm(h, eps=eps)
        e = widen_bf16(emb[t]) if emb.dtype == np.uint16 else _f32(emb[t])
        _, eb = rmsnorm(e, eps=eps)
        x = np.concatenate([widen_bf16(hb), widen_bf16(eb)], axis=1)
        u = lm_head(x, w_proj)
        _, ub = rmsnorm(u, eps=eps)
        y = expert_ffn_routed(widen_bf16(ub), wgu, wd, np.array([0, B], np.int32), rows, 1)
        h = combine(y, None, rows[:, None], np.ones((B, 1), np.float32), u)
        _, xb = rmsnorm(h, eps=eps)
        z = widen_bf16(bf16_round(lm_head(widen_bf16(xb), w_lm)))
        t = verify_greedy(z[:, None, :], np.zeros((B, 0), np.int32))[0][:, 0].astype(np.int32)
        drafts[:, i] = t
    return drafts, h

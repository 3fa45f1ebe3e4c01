"""Thin ctypes binding of libmoespec.so (include/moespec.h).

Argument marshalling only: tensors are torch CUDA tensors, passed by
data_ptr() together with the current CUDA stream; every step runs in the
library's kernels.  There is no fallback: if the shared library is missing
or fails to load, importing this module raises.  Build it with
`python -m speculative_decoding_verification_router_b200.build`.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoespec.so")

MS_F32, MS_BF16 = 0, 1
STATUS = {0: "MS_OK", -1: "MS_ERR_INVALID_ARG", -2: "MS_ERR_UNSUPPORTED", -3: "MS_ERR_WORKSPACE",
          -4: "MS_ERR_CUDA", -5: "MS_ERR_TIMEOUT", -6: "MS_ERR_DEVICE_INDEX",
          -7: "MS_ERR_DRAIN_TIMEOUT"}


class MoeSpecError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        msg = f"{where}: {STATUS.get(code, code)}"
        if code == -4:
            msg += f" ({_lib.ms_last_cuda_error_string().decode()})"
        super().__init__(msg)


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libmoespec.so not built at {_LIB_PATH}; run "
                          "`python -m speculative_decoding_verification_router_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, F, Z, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t, ctypes.c_uint64
    sig = {
        "moe_rmsnorm": (I, [P, P, I, I, F, P, P]),
        "moe_route_topk": (I, [P, P, P, I, I, I, I, I, P, P, P]),
        "moe_route_topk_tensor_workspace_size": (Z, [I, I]),
        "moe_route_topk_tensor": (I, [P, P, P, I, I, I, I, I, P, P, P, Z, P]),
        "moe_permute_workspace_size": (Z, [I, I, I]),
        "moe_permute": (I, [P, I, I, I, P, P, P, P, Z, P]),
        "moe_expert_ffn_workspace_size": (Z, [I, I, I, I, I, I]),
        "moe_expert_ffn": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, P, I, P, P, Z, P]),
        "moe_combine": (I, [P, I, P, P, P, P, I, I, I, P, P, P]),
        "lm_head_workspace_size": (Z, [I, I, I]),
        "lm_head_logits": (I, [P, P, I, I, I, P, P, Z, P]),
        "spec_verify_workspace_size": (Z, [I, I, I]),
        "spec_verify_greedy": (I, [P, I, P, I, I, I, P, P, P, P, Z, P]),
        "spec_verify_lm_head_workspace_size": (Z, [I, I, I, I]),
        "fastmtp_draft_workspace_size": (Z, [I, I, I, I]),
        "fastmtp_draft": (I, [P, P, P, P, P, P, P, I, I, I, I, I, P, P, P, Z, P]),
        "spec_verify_lm_head_greedy": (I, [P, P, P, I, I, I, I, P, P, P, P, Z, P]),
        "moe_layer_workspace_size": (Z, [I, I, I, I, I, I]),
        "moe_layer_forward": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, Z, P]),
        "ms_device_status": (I, [P, P]),
        "ms_set_wait_limit_ns": (None, [U64]),
        "ms_get_wait_limit_ns": (U64, []),
        "ms_debug_bounded_wait": (I, [P, I, P, P]),
        "ms_trace_enable": (I, [I]),
        "ms_trace_disable": (None, []),
        "ms_trace_reset": (None, []),
        "ms_trace_count": (I, []),
        "ms_trace_read": (I, [I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(F)]),
        "ms_status_string": (ctypes.c_char_p, [I]),
        "ms_last_cuda_error_string": (ctypes.c_char_p, []),
        "ms_version": (I, []),
        "moe_pack_weights": (I, [P, I, I, I, P, P]),
        "ms_set_device_trace": (I, [P, Z]),
        "ms_set_batch_invariant": (None, [I]),
        "ms_get_batch_invariant": (I, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib():
    return _lib


# ------------------------------------------------------------------ helpers

def _p(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, where: str):
    if code != 0:
        raise MoeSpecError(code, where)


def _dev(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


class Workspace:
    """A reusable, 1024-byte aligned device scratch buffer."""

    def __init__(self, nbytes: int, device=None):
        self.nbytes = int(nbytes)
        self._buf = torch.empty(self.nbytes + 1024, dtype=torch.uint8, device=device or "cuda")
        base = self._buf.data_ptr()
        self.offset = (-base) % 1024
        self.ptr = base + self.offset

    def c(self):
        return ctypes.c_void_p(self.ptr)

    def view(self) -> torch.Tensor:
        return self._buf[self.offset: self.offset + self.nbytes]


def _ws(ws: Optional[Workspace], need: int, device) -> Workspace:
    if ws is not None and ws.nbytes >= need:
        return ws
    return Workspace(max(need, 1), device)


class CapturedStep:
    """A fixed sequence of calls of this library (and the host<->device copies
    around them) captured once into a CUDA graph and replayed as one launch,
    for decode loops whose per-step host launch cost would otherwise exceed
    the device time.  `fn` must use preallocated tensors and workspaces (the
    graph replays the same addresses); it is run `warmup` times on `stream`
    before capture.  Every library call launches its kernels on the current
    stream, so the captured calls must not name another stream."""

    def __init__(self, fn, stream=None, warmup: int = 2):
        self.stream = stream or torch.cuda.Stream()
        with torch.cuda.stream(self.stream):
            for _ in range(warmup):
                fn()
        torch.cuda.synchronize()
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph, stream=self.stream):
            fn()
        torch.cuda.synchronize()

    def __call__(self):
        with torch.cuda.stream(self.stream):
            self.graph.replay()


# ------------------------------------------------------------------ calls

def pack_weights(w: torch.Tensor, stream=None) -> torch.Tensor:
    """Repack a bf16 weight stack [n, rows, cols] (or [rows, cols]) into the
    tile-contiguous layout the GEMM entry points read.  Same shape and dtype;
    only the element order changes."""
    _dev(w, torch.bfloat16, "w")
    shape = w.shape
    w3 = w.view(1, *shape) if w.dim() == 2 else w
    n, rows, cols = w3.shape
    out = torch.empty_like(w)
    _check(_lib.moe_pack_weights(_p(w3), n, rows, cols, _p(out), _stream(stream)), "moe_pack_weights")
    return out


def rmsnorm(a: torch.Tensor, gamma=None, eps: float = 1e-6, out=None, stream=None) -> torch.Tensor:
    _dev(a, torch.float32, "a")
    T, H = a.shape
    out = out if out is not None else torch.empty((T, H), dtype=torch.bfloat16, device=a.device)
    _check(_lib.moe_rmsnorm(_p(a), _p(gamma), T, H, eps, _p(out), _stream(stream)), "moe_rmsnorm")
    return out


def route_topk(xhat: torch.Tensor, w_router: torch.Tensor, bias=None, k: int = 6,
               renormalize: bool = False, out=None, stream=None):
    _dev(xhat, torch.bfloat16, "xhat")
    _dev(w_router, torch.float32, "w_router")
    if bias is not None:
        _dev(bias, torch.float32, "bias")
    T, H = xhat.shape
    E = w_router.shape[0]
    idx, w = out if out is not None else (torch.empty((T, k), dtype=torch.int32, device=xhat.device),
                                          torch.empty((T, k), dtype=torch.float32, device=xhat.device))
    _check(_lib.moe_route_topk(_p(xhat), _p(w_router), _p(bias), T, H, E, k, int(renormalize),
                               _p(idx), _p(w), _stream(stream)), "moe_route_topk")
    return idx, w


def route_topk_tensor(xhat: torch.Tensor, w_router: torch.Tensor, bias=None, k: int = 6,
                      renormalize: bool = False, ws: Optional[Workspace] = None, out=None, stream=None):
    """The router on the tensor cores (prefill-sized batches): same results as route_topk."""
    _dev(xhat, torch.bfloat16, "xhat")
    _dev(w_router, torch.float32, "w_router")
    if bias is not None:
        _dev(bias, torch.float32, "bias")
    T, H = xhat.shape
    E = w_router.shape[0]
    idx, w = out if out is not None else (torch.empty((T, k), dtype=torch.int32, device=xhat.device),
                                          torch.empty((T, k), dtype=torch.float32, device=xhat.device))
    wsb = _ws(ws, _lib.moe_route_topk_tensor_workspace_size(E, H), xhat.device)
    _check(_lib.moe_route_topk_tensor(_p(xhat), _p(w_router), _p(bias), T, H, E, k, int(renormalize), _p(idx), _p(w),
                                      wsb.c(), wsb.nbytes, _stream(stream)), "moe_route_topk_tensor")
    return idx, w


def permute(idx: torch.Tensor, E: int, ws: Optional[Workspace] = None, out=None, stream=None):
    _dev(idx, torch.int32, "topk_idx")
    T, k = idx.shape
    dev = idx.device
    off, perm, slot = out if out is not None else (
        torch.empty(E + 1, dtype=torch.int32, device=dev),
        torch.empty(T * k, dtype=torch.int32, device=dev),
        torch.empty((T, k), dtype=torch.int32, device=dev))
    need = _lib.moe_permute_workspace_size(T, k, E)
    w = _ws(ws, need, dev) if need > 0 else ws
    _check(_lib.moe_permute(_p(idx), T, k, E, _p(off), _p(perm), _p(slot),
                            w.c() if w is not None else None, w.nbytes if w is not None else 0,
                            _stream(stream)), "moe_permute")
    return off, perm, slot


def expert_ffn_workspace_size(T, H, E, I, S, k) -> int:
    return _lib.moe_expert_ffn_workspace_size(T, H, E, I, S, k)


def expert_ffn(xhat, offsets, perm, w_gate_up, w_down, ws_gate_up=None, ws_down=None, k: int = 6,
               y_dtype=torch.float32, ws: Optional[Workspace] = None, out=None, stream=None):
    _dev(xhat, torch.bfloat16, "xhat")
    _dev(w_gate_up, torch.bfloat16, "w_gate_up")
    _dev(w_down, torch.bfloat16, "w_down")
    T, H = xhat.shape
    E, twoI, _ = w_gate_up.shape
    I = twoI // 2
    S = 0 if ws_gate_up is None else ws_gate_up.shape[0]
    dev = xhat.device
    if out is None:
        y = torch.empty((T * k, H), dtype=y_dtype, device=dev)
        ysh = torch.empty((T, H), dtype=torch.float32, device=dev) if S > 0 else None
    else:
        y, ysh = out
    w = _ws(ws, expert_ffn_workspace_size(T, H, E, I, S, k), dev)
    _check(_lib.moe_expert_ffn(_p(xhat), _p(offsets), _p(perm), _p(w_gate_up), _p(w_down), _p(ws_gate_up),
                               _p(ws_down), T, H, E, I, S, k, _p(y),
                               MS_BF16 if y.dtype == torch.bfloat16 else MS_F32, _p(ysh), w.c(), w.nbytes,
                               _stream(stream)), "moe_expert_ffn")
    return y, ysh


def combine(y_perm, y_shared, slot_of, topk_w, residual, out=None, out_bf16=None, stream=None):
    T, k = slot_of.shape
    H = y_perm.shape[1]
    out = out if out is not None else torch.empty((T, H), dtype=torch.float32, device=y_perm.device)
    ydt = MS_BF16 if y_perm.dtype == torch.bfloat16 else MS_F32
    _check(_lib.moe_combine(_p(y_perm), ydt, _p(y_shared), _p(slot_of), _p(topk_w), _p(residual), T, H, k,
                            _p(out), _p(out_bf16), _stream(stream)), "moe_combine")
    return out


def lm_head(xhat, w_lm, ws: Optional[Workspace] = None, out=None, stream=None):
    _dev(xhat, torch.bfloat16, "xhat")
    _dev(w_lm, torch.bfloat16, "w_lm")
    T, H = xhat.shape
    V = w_lm.shape[0]
    out = out if out is not None else torch.empty((T, V), dtype=torch.bfloat16, device=xhat.device)
    w = _ws(ws, _lib.lm_head_workspace_size(T, H, V), xhat.device)
    _check(_lib.lm_head_logits(_p(xhat), _p(w_lm), T, H, V, _p(out), w.c(), w.nbytes, _stream(stream)),
           "lm_head_logits")
    return out


def verify_greedy(logits, draft, ws: Optional[Workspace] = None, out=None, stream=None):
    B, K1, V = logits.shape
    K = K1 - 1
    _dev(draft, torch.int32, "draft")
    dt = MS_BF16 if logits.dtype == torch.bfloat16 else MS_F32
    if dt == MS_F32:
        _dev(logits, torch.float32, "logits")
    dev = logits.device
    am, cm, n = out if out is not None else (torch.empty((B, K1), dtype=torch.int32, device=dev),
                                             torch.empty((B, K1), dtype=torch.int32, device=dev),
                                             torch.empty(B, dtype=torch.int32, device=dev))
    w = _ws(ws, _lib.spec_verify_workspace_size(B, K, V), dev)
    _check(_lib.spec_verify_greedy(_p(logits), dt, _p(draft), B, K, V, _p(am), _p(cm), _p(n), w.c(), w.nbytes,
                                   _stream(stream)), "spec_verify_greedy")
    return am, cm, n


def verify_lm_head_greedy(xhat, w_lm, draft, ws: Optional[Workspace] = None, out=None, stream=None):
    """Vocab head with the verification's argmax fused into its epilogue, then
    the prefix match.  xhat [B*(K+1), H] bf16, w_lm packed [V, H] bf16, draft [B, K] int32."""
    _dev(xhat, torch.bfloat16, "xhat")
    _dev(w_lm, torch.bfloat16, "w_lm")
    _dev(draft, torch.int32, "draft")
    B, K = draft.shape
    T, H = xhat.shape
    V = w_lm.shape[0]
    if T != B * (K + 1):
        raise ValueError(f"xhat has {T} rows, expected B*(K+1) = {B * (K + 1)}")
    dev = xhat.device
    am, cm, n = out if out is not None else (torch.empty((B, K + 1), dtype=torch.int32, device=dev),
                                             torch.empty((B, K + 1), dtype=torch.int32, device=dev),
                                             torch.empty(B, dtype=torch.int32, device=dev))
    w = _ws(ws, _lib.spec_verify_lm_head_workspace_size(B, K, H, V), dev)
    _check(_lib.spec_verify_lm_head_greedy(_p(xhat), _p(w_lm), _p(draft), B, K, H, V, _p(am), _p(cm), _p(n),
                                           w.c(), w.nbytes, _stream(stream)), "spec_verify_lm_head_greedy")
    return am, cm, n


def fastmtp_draft(h0, tok0, emb, w_proj, w_gate_up, w_down, w_lm, K: int, ws: Optional[Workspace] = None,
                  out=None, stream=None):
    """FastMTP draft block applied K times on the device.  h0 [B,H] fp32, tok0 [B]
    int32, emb [V,H] bf16 (row-major), w_proj [H,2H], w_gate_up [2I,H], w_down [H,I],
    w_lm [V,H] bf16 packed by pack_weights.  Returns (drafts [B,K] int32, h_out [B,H] fp32)."""
    _dev(h0, torch.float32, "h0")
    _dev(tok0, torch.int32, "tok0")
    for name, t in (("emb", emb), ("w_proj", w_proj), ("w_gate_up", w_gate_up), ("w_down", w_down), ("w_lm", w_lm)):
        _dev(t, torch.bfloat16, name)
    B, H = h0.shape
    V = emb.shape[0]
    I = w_down.shape[-1]
    dev = h0.device
    drafts, h_out = out if out is not None else (torch.empty((B, K), dtype=torch.int32, device=dev),
                                                 torch.empty((B, H), dtype=torch.float32, device=dev))
    w = _ws(ws, _lib.fastmtp_draft_workspace_size(B, H, I, V), dev)
    _check(_lib.fastmtp_draft(_p(h0), _p(tok0), _p(emb), _p(w_proj), _p(w_gate_up), _p(w_down), _p(w_lm), B, H, I,
                              V, K, _p(drafts), _p(h_out), w.c(), w.nbytes, _stream(stream)), "fastmtp_draft")
    return drafts, h_out


def layer_workspace_size(T, H, E, I, S, k) -> int:
    return _lib.moe_layer_workspace_size(T, H, E, I, S, k)


def layer_forward(a, w_router, bias, w_gate_up, w_down, ws_gate_up, ws_down, k: int,
                  renormalize: bool = False, ws: Optional[Workspace] = None, out=None, stream=None):
    _dev(a, torch.float32, "a")
    T, H = a.shape
    E, twoI, _ = w_gate_up.shape
    I = twoI // 2
    S = 0 if ws_gate_up is None else ws_gate_up.shape[0]
    out = out if out is not None else torch.empty((T, H), dtype=torch.float32, device=a.device)
    w = _ws(ws, layer_workspace_size(T, H, E, I, S, k), a.device)
    _check(_lib.moe_layer_forward(_p(a), _p(w_router), _p(bias), _p(w_gate_up), _p(w_down), _p(ws_gate_up),
                                  _p(ws_down), T, H, E, I, S, k, int(renormalize), _p(out), w.c(), w.nbytes,
                                  _stream(stream)), "moe_layer_forward")
    return out


def device_status(ws: Workspace, stream=None) -> int:
    """Synchronise, return and clear the device status word kept in `ws`."""
    return int(_lib.ms_device_status(ws.c(), _stream(stream)))


def set_batch_invariant(on: bool):
    """Process-wide: batch-invariant GEMM schedules for the calls that follow
    (see ms_set_batch_invariant in include/moespec.h)."""
    _lib.ms_set_batch_invariant(int(bool(on)))


def get_batch_invariant() -> bool:
    return bool(_lib.ms_get_batch_invariant())


def set_wait_limit_ns(ns: int):
    _lib.ms_set_wait_limit_ns(int(ns))


def get_wait_limit_ns() -> int:
    return int(_lib.ms_get_wait_limit_ns())


def debug_bounded_wait(flag: torch.Tensor, expect: int, status: torch.Tensor, stream=None):
    _check(_lib.ms_debug_bounded_wait(_p(flag), int(expect), _p(status), _stream(stream)), "ms_debug_bounded_wait")


def set_device_trace(buf: Optional[torch.Tensor]):
    """Point the GEMMs' per-CTA timeline at `buf` (uint64 tensor, >= 8*256*8), or None to stop."""
    if buf is None:
        _check(_lib.ms_set_device_trace(None, 0), "ms_set_device_trace")
    else:
        _check(_lib.ms_set_device_trace(_p(buf), buf.numel() * buf.element_size()), "ms_set_device_trace")


def trace_enable(capacity: int):
    _check(_lib.ms_trace_enable(int(capacity)), "ms_trace_enable")


def trace_disable():
    _lib.ms_trace_disable()


def trace_reset():
    _lib.ms_trace_reset()


def trace_records():
    """[(kernel_name, milliseconds)] for every traced launch (after a synchronize)."""
    out = []
    for i in range(_lib.ms_trace_count()):
        name = ctypes.c_char_p()
        ms = ctypes.c_float()
        _check(_lib.ms_trace_read(i, ctypes.byref(name), ctypes.byref(ms)), "ms_trace_read")
        out.append((name.value.decode(), ms.value))
    return out


# ------------------------------------------------------------------ conversions

def bf16_from_bits(bits, device="cuda") -> torch.Tensor:
    """uint16 numpy array of bf16 bit patterns -> torch.bfloat16 tensor on `device`."""
    import numpy as np
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def bf16_to_bits(t: torch.Tensor):
    """torch.bfloat16 tensor -> uint16 numpy bit patterns (host)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view("uint16")

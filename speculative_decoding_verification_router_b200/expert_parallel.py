"""Expert-parallel MoE layer over R ranks, one GPU each.

The decoder layer of the pages has 64 routed and two shared SwiGLU experts
with top-6 routing (clawpit.io, "Lean architecture with a compressed
encoder").  Spread over R ranks:

* routed experts: rank r owns the contiguous block [r E/R, (r+1) E/R);
* shared experts: two SwiGLU experts equal one expert whose intermediate
  features are the two concatenated, and a SwiGLU expert's output is the sum
  over its intermediate features of (down column) x (feature's activation);
  so the S*I concatenated features are split into contiguous blocks of 128,
  rank r taking its share, and the ranks' partial outputs add up to the
  shared experts' output.

Two forms of the layer:

* `decode_layer` (verify-sized batches, every rank holds all T tokens): each
  rank normalises and routes all tokens (the routing is per-token and
  identical on every rank), computes the rows of its own experts and its
  block of shared features, combines those into a partial layer output (the
  residual on rank 0 only), and one all-reduce (sum) over the ranks gives
  every rank the layer output.  Data on the wire: T*H fp32 per rank.
* `prefill_layer` (each rank holds its own tokens): each rank routes its
  tokens, sends each (token, slot) row to the rank that owns its expert (an
  all-to-all, counts first), the owner runs its experts on what it received
  (regrouped by expert) and sends the results back (a second all-to-all); the
  shared experts run on every rank for its own tokens (token-parallel), and
  the combine is local.

Collectives are torch.distributed (NCCL over NVLink on GPUs, gloo on CPUs);
no TMA multicast is involved.  The per-rank compute goes through a backend
object: `LibraryBackend` runs every step in this library's kernels; the
row gathers and regrouping around the all-to-all are index plumbing done with
torch ops.  Not measured on hardware: every run available to this build had
one GPU.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch
import torch.distributed as dist

SHARED_BLOCK = 128   # the expert GEMMs take intermediate widths in multiples of 128


@dataclasses.dataclass(frozen=True)
class Partition:
    """Which routed experts and which shared intermediate features rank `rank` of `R` owns."""
    E: int
    S: int
    I: int
    R: int
    rank: int

    def __post_init__(self):
        if self.E % self.R != 0:
            raise ValueError(f"E={self.E} experts do not split evenly over R={self.R} ranks")
        if (self.S * self.I) % SHARED_BLOCK != 0:
            raise ValueError("the shared experts' width must be a multiple of 128")

    @property
    def experts_per_rank(self) -> int:
        return self.E // self.R

    @property
    def e0(self) -> int:
        return self.rank * self.experts_per_rank

    def owner(self, e):
        """Rank owning routed expert e (works on numpy arrays)."""
        return e // self.experts_per_rank

    def shared_cols(self, rank: Optional[int] = None):
        """[c0, c1): the concatenated shared features of `rank` (blocks of 128 dealt in order)."""
        r = self.rank if rank is None else rank
        nb = (self.S * self.I) // SHARED_BLOCK
        return (r * nb // self.R) * SHARED_BLOCK, ((r + 1) * nb // self.R) * SHARED_BLOCK


def shared_as_one_expert(ws_gate_up, ws_down):
    """The S shared experts as one SwiGLU expert of width S*I: ([2SI, H], [H, SI])
    (gate rows of all experts, then their up rows; down columns in the same order)."""
    S, twoI, _ = ws_gate_up.shape
    I = twoI // 2
    gate = np.concatenate([ws_gate_up[s, :I] for s in range(S)], axis=0)
    up = np.concatenate([ws_gate_up[s, I:] for s in range(S)], axis=0)
    down = np.concatenate([ws_down[s] for s in range(S)], axis=1)
    return np.concatenate([gate, up], axis=0), down


def shard_layer(w_gate_up, w_down, ws_gate_up, ws_down, part: Partition):
    """This rank's weights of one layer (host arrays, bf16 bits or fp32):
    routed [E/R, 2I, H] / [E/R, H, I]; its block of shared features as one
    dense expert [1, 2w, H] / [1, H, w] (w = 0 when the rank has none); and
    the whole shared experts as one dense expert (the prefill form runs them
    token-parallel)."""
    e0, e1 = part.e0, part.e0 + part.experts_per_rank
    gu, d = shared_as_one_expert(ws_gate_up, ws_down)
    SI = gu.shape[0] // 2
    c0, c1 = part.shared_cols()
    sh_gu = np.concatenate([gu[c0:c1], gu[SI + c0:SI + c1]], axis=0)[None]
    sh_d = np.ascontiguousarray(d[:, c0:c1])[None]
    return dict(w_gate_up=np.ascontiguousarray(w_gate_up[e0:e1]), w_down=np.ascontiguousarray(w_down[e0:e1]),
                shared_gate_up=sh_gu, shared_down=sh_d, width=c1 - c0,
                all_shared_gate_up=gu[None], all_shared_down=np.ascontiguousarray(d)[None])


# ---------------------------------------------------------------- drivers

def decode_layer(be, part: Partition, a, w_router, local, k: int, bias=None, group=None):
    """Layer output [T, H] fp32 on every rank, from the same T tokens on every rank."""
    xh = be.rmsnorm(a)
    idx, w = be.route(xh, w_router, bias, k)
    off, perm, slot = be.permute(idx, part.E)
    # this rank's experts: the routing offsets of its block (absolute rows of
    # the full grouping); rows of other ranks' experts stay zero
    y = be.expert_ffn(xh, be.offsets_slice(off, part.e0, part.experts_per_rank + 1), perm,
                      local["w_gate_up"], local["w_down"], k)
    ysh = be.dense_ffn(xh, local["shared_gate_up"], local["shared_down"]) if local["width"] > 0 else None
    out = be.combine(y, ysh, slot, w, a if part.rank == 0 else None)
    out_t = be.to_torch(out)
    dist.all_reduce(out_t, group=group)   # the sum of the ranks' partial outputs
    return out_t


def prefill_layer(be, part: Partition, a_local, w_router, local, k: int, group=None):
    """Layer output [T_r, H] for this rank's own T_r tokens."""
    R, E, epr = part.R, part.E, part.experts_per_rank
    dv = be.device
    xh = be.rmsnorm(a_local)
    idx, w = be.route(xh, w_router, None, k)
    off, perm, slot = be.permute(idx, E)
    off_h = be.to_host_int(off).astype(np.int64)
    # rows in expert order are grouped by owner too (each rank's experts are contiguous)
    send = np.array([off_h[(d + 1) * epr] - off_h[d * epr] for d in range(R)], np.int64)
    expert_of_row = np.repeat(np.arange(E, dtype=np.int64), np.diff(off_h))
    recv = torch.empty(R, dtype=torch.int64, device=dv)
    dist.all_to_all_single(recv, torch.from_numpy(send).to(dv), group=group)
    send_l, recv_l = send.tolist(), recv.cpu().tolist()
    n = int(sum(recv_l))
    x_rows = be.rows_to_torch(be.gather_rows(xh, perm))                       # [T_r*k, H] expert order
    x_recv = x_rows.new_empty((n,) + tuple(x_rows.shape[1:]))
    dist.all_to_all_single(x_recv, x_rows, recv_l, send_l, group=group)
    id_send = torch.from_numpy((expert_of_row % epr).astype(np.int32)).to(dv)
    id_recv = torch.empty(n, dtype=torch.int32, device=dv)
    dist.all_to_all_single(id_recv, id_send, recv_l, send_l, group=group)
    # the owner: regroup what it received by its experts, run them, restore the order
    order = torch.argsort(id_recv, stable=True)
    cnt = torch.bincount(id_recv.long(), minlength=epr).cpu().numpy()
    off_r = np.concatenate([[0], np.cumsum(cnt)]).astype(np.int32)
    y_sorted = be.to_torch(be.expert_ffn(be.rows_from_torch(x_recv[order]), be.from_host_int(off_r),
                                         be.from_host_int(np.arange(n, dtype=np.int32)), local["w_gate_up"],
                                         local["w_down"], 1))
    y_recv = torch.empty_like(y_sorted)
    y_recv[order] = y_sorted
    y_back = y_recv.new_empty((int(sum(send_l)),) + tuple(y_recv.shape[1:]))
    dist.all_to_all_single(y_back, y_recv, send_l, recv_l, group=group)     # rows back to their tokens' rank
    ysh = be.dense_ffn(xh, local["all_shared_gate_up"], local["all_shared_down"])
    return be.to_torch(be.combine(be.from_torch(y_back), ysh, slot, w, a_local))


# ---------------------------------------------------------------- the library as the backend

class LibraryBackend:
    """Every compute step in this library's kernels (CUDA tensors); weights
    are packed once by `load`."""

    device = "cuda"

    def __init__(self):
        from . import moespec
        self.ms = moespec

    def load(self, local):
        """Device copies of `shard_layer`'s arrays, packed for the GEMMs."""
        ms = self.ms
        dev = lambda a: ms.bf16_from_bits(a) if a.dtype == np.uint16 else torch.from_numpy(a).cuda()
        out = dict(local)
        for key in ("w_gate_up", "w_down", "shared_gate_up", "shared_down", "all_shared_gate_up", "all_shared_down"):
            if local[key].size:
                out[key] = ms.pack_weights(dev(local[key]))
        return out

    def rmsnorm(self, a):
        return self.ms.rmsnorm(a)

    def route(self, xh, w_router, bias, k):
        return self.ms.route_topk(xh, w_router, bias, k)

    def permute(self, idx, E):
        return self.ms.permute(idx, E)

    def offsets_slice(self, off, e0, n):
        return off[e0:e0 + n]

    def expert_ffn(self, xh, off, perm, wgu, wd, k):
        T, H = xh.shape
        y = torch.zeros((T * k, H), dtype=torch.float32, device=xh.device)
        self.ms.expert_ffn(xh, off, perm, wgu, wd, None, None, k, out=(y, None))
        return y

    def dense_ffn(self, xh, wgu, wd):
        T, H = xh.shape
        dev = xh.device
        off = torch.tensor([0, T], dtype=torch.int32, device=dev)
        perm = torch.arange(T, dtype=torch.int32, device=dev)
        y = torch.empty((T, H), dtype=torch.float32, device=dev)
        self.ms.expert_ffn(xh, off, perm, wgu, wd, None, None, 1, out=(y, None))
        return y

    def combine(self, y, ysh, slot, w, residual):
        return self.ms.combine(y, ysh, slot, w, residual)

    def gather_rows(self, xh, perm):
        return xh[perm.long()]

    def rows_to_torch(self, x):
        return x

    def rows_from_torch(self, x):
        return x.contiguous()

    def to_torch(self, x):
        return x

    def from_torch(self, x):
        return x.contiguous()

    def to_host_int(self, t):
        return t.cpu().numpy()

    def from_host_int(self, a):
        return torch.from_numpy(np.ascontiguousarray(a, np.int32)).cuda()

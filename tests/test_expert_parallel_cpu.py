"""The expert-parallel layer's partitioning, dispatch and combine on CPU.

Two or four gloo ranks run speculative_decoding_verification_router_b200.expert_parallel
with the oracle as the per-rank compute backend (the collectives and the
index plumbing are the module's own); the result must equal the oracle's
single-process layer on the whole batch up to fp32 rounding of the different
summation order.  The decode form keeps every token on every rank and
all-reduces partial layer outputs (routed experts by owner, shared experts
by blocks of intermediate features); the prefill form sends each
(token, slot) row to its expert's owner and back (all-to-all)."""
import os
import socket
import sys

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
T, H, E, I, K_TOP, S = 24, 128, 8, 128, 2, 2


def _shape():
    from speculative_decoding_verification_router_b200 import synth
    return synth.MoEShape("ep_cpu", B=1, K=0, H=H, E=E, I=I, k=K_TOP, S=S, V=256, router_std=0.3,
                          weight_std=0.1, tokens=T)


class OracleBackend:
    """The oracle as the compute of one rank (bf16 activations as uint16 bits)."""
    device = "cpu"

    def __init__(self):
        import oracle
        self.o = oracle

    def rmsnorm(self, a):
        return self.o.rmsnorm(a)[1]

    def route(self, xh, w_router, bias, k):
        idx, w, _, _ = self.o.route_topk(self.o.widen_bf16(xh), w_router, bias, k)
        return idx, w

    def permute(self, idx, E_):
        return self.o.permute(idx, E_)

    def offsets_slice(self, off, e0, n):
        return np.ascontiguousarray(off[e0:e0 + n])

    def expert_ffn(self, xh, off, perm, wgu, wd, k):
        # rows of groups outside `off` are not computed (NaN): zero, as on the GPU
        y = self.o.expert_ffn_routed(self.o.widen_bf16(xh), wgu, wd, off, perm, k)
        return np.where(np.isnan(y), np.float32(0), y)

    def dense_ffn(self, xh, wgu, wd):
        return self.o.expert_ffn_shared(self.o.widen_bf16(xh), wgu, wd)

    def combine(self, y, ysh, slot, w, residual):
        return self.o.combine(y, ysh, slot, w, residual)

    def gather_rows(self, xh, perm):
        return np.ascontiguousarray(xh[perm])

    # gloo moves no 16-bit types: the bf16 rows travel as their exact fp32 widening
    def rows_to_torch(self, x):
        import torch
        return torch.from_numpy(self.o.widen_bf16(x).copy())

    def rows_from_torch(self, t):
        return (t.contiguous().numpy().view(np.uint32) >> np.uint32(16)).astype(np.uint16)

    def to_torch(self, x):
        import torch
        return torch.from_numpy(np.ascontiguousarray(x, np.float32).copy())

    def from_torch(self, t):
        return t.contiguous().numpy()

    def to_host_int(self, t):
        return np.asarray(t)

    def from_host_int(self, a):
        return np.ascontiguousarray(a, np.int32)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir, mode):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from speculative_decoding_verification_router_b200 import expert_parallel as ep, synth
    shp = _shape()
    lw = synth.layer_weights(shp, 0)
    a = synth.normal(0, "ep_cpu.a", (T, H), 1.0)
    part = ep.Partition(E, S, I, world, rank)
    local = ep.shard_layer(lw.w_gate_up, lw.w_down, lw.ws_gate_up, lw.ws_down, part)
    be = OracleBackend()
    if mode == "decode":
        out = ep.decode_layer(be, part, a, lw.w_router, local, K_TOP).numpy()
    else:
        lo, hi = rank * T // world, (rank + 1) * T // world
        out = ep.prefill_layer(be, part, np.ascontiguousarray(a[lo:hi]), lw.w_router, local, K_TOP).numpy()
    np.save(os.path.join(out_dir, f"{mode}{rank}.npy"), out)
    dist.barrier()
    dist.destroy_process_group()


def _reference():
    sys.path.insert(0, ROOT)
    import oracle
    from speculative_decoding_verification_router_b200 import synth
    shp = _shape()
    lw = synth.layer_weights(shp, 0)
    a = synth.normal(0, "ep_cpu.a", (T, H), 1.0)
    return oracle.moe_layer(a, lw, K_TOP)["out"]


def _close(got, ref):
    d = np.abs(got.astype(np.float64) - ref.astype(np.float64))
    assert d.max() <= 1e-5 * max(np.abs(ref).max(), 1.0), d.max()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("mode", ["decode", "prefill"])
def test_ranks_equal_the_whole_layer(tmp_path, mode, world):
    # with 4 ranks the 2 x 128 shared features go to ranks 1 and 3 only:
    # ranks 0 and 2 hold no shared block and contribute routed rows alone
    import oracle
    oracle.build()
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path), mode), nprocs=world, join=True,
                       start_method="spawn")
    ref = _reference()
    if mode == "decode":
        for r in range(world):
            _close(np.load(tmp_path / f"decode{r}.npy"), ref)
    else:
        got = np.concatenate([np.load(tmp_path / f"prefill{r}.npy") for r in range(world)])
        _close(got, ref)


def test_partition_covers_every_expert_and_shared_feature_once():
    sys.path.insert(0, ROOT)
    from speculative_decoding_verification_router_b200 import expert_parallel as ep
    for (E_, S_, I_, R) in [(64, 2, 896, 8), (64, 2, 896, 2), (8, 2, 128, 2), (64, 2, 896, 1)]:
        experts = np.concatenate([np.arange(ep.Partition(E_, S_, I_, R, r).e0,
                                            ep.Partition(E_, S_, I_, R, r).e0 + E_ // R) for r in range(R)])
        np.testing.assert_array_equal(experts, np.arange(E_))
        cols = [ep.Partition(E_, S_, I_, R, r).shared_cols() for r in range(R)]
        assert cols[0][0] == 0 and cols[-1][1] == S_ * I_
        assert all(cols[r][1] == cols[r + 1][0] for r in range(R - 1))
        assert all((c1 - c0) % 128 == 0 for c0, c1 in cols)
        for e in range(E_):
            assert ep.Partition(E_, S_, I_, R, 0).owner(e) == e // (E_ // R)


def test_shared_experts_as_one_expert_is_exact():
    # two SwiGLU experts = one expert with the intermediate features concatenated,
    # and its column blocks sum to the whole (the split the decode form uses)
    sys.path.insert(0, ROOT)
    import oracle
    from speculative_decoding_verification_router_b200 import expert_parallel as ep, synth
    shp = _shape()
    lw = synth.layer_weights(shp, 1)
    x = oracle.widen_bf16(synth.normal_bf16(1, "ep_cpu.x", (8, H), 1.0))
    ref = oracle.expert_ffn_shared(x, lw.ws_gate_up, lw.ws_down)
    gu, d = ep.shared_as_one_expert(lw.ws_gate_up, lw.ws_down)
    one = oracle.expert_ffn_shared(x, gu[None], d[None])
    _close(one, ref)
    parts = []
    for r in range(2):
        loc = ep.shard_layer(lw.w_gate_up, lw.w_down, lw.ws_gate_up, lw.ws_down, ep.Partition(E, S, I, 2, r))
        parts.append(oracle.expert_ffn_shared(x, loc["shared_gate_up"], loc["shared_down"]))
    _close(parts[0] + parts[1], ref)

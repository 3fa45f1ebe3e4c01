"""The expert-parallel layer's GPU backend on one GPU (a one-rank NCCL group):
the decode form (partial outputs all-reduced) and the prefill form (rows
dispatched to their expert's owner and back by all-to-all) run every compute
step in the library and must match the oracle's layer within the layer
tolerance.  With one rank the collectives move nothing; the multi-rank index
arithmetic is tested with two gloo ranks in test_expert_parallel_cpu.py."""
import datetime
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import oracle
from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import assert_close, dev, host
from tests.inputs import routed_layer_inputs

pytestmark = pytest.mark.gpu


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.fixture(scope="module")
def group():
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_port()}", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60))
    yield None
    dist.destroy_process_group()


@pytest.mark.parametrize("mode,shp", [("decode", synth.VERIFY_B1), ("decode", synth.VERIFY_B32),
                                      ("prefill", synth.MoEShape("ep_prefill", B=1, K=0, H=1280, E=64, I=896, k=6,
                                                                 S=2, V=129280, router_std=0.05, tokens=300))],
                         ids=["decode_b1", "decode_b32", "prefill_t300"])
def test_expert_parallel_one_rank_matches_oracle(group, mode, shp):
    from speculative_decoding_verification_router_b200 import expert_parallel as ep
    a, lw, bias = routed_layer_inputs(shp, 0)
    ref = oracle.moe_layer(a, lw, shp.k, bias if mode == "decode" else None)
    part = ep.Partition(shp.E, shp.S, shp.I, 1, 0)
    be = ep.LibraryBackend()
    local = be.load(ep.shard_layer(lw.w_gate_up, lw.w_down, lw.ws_gate_up, lw.ws_down, part))
    wr = dev(lw.w_router)
    if mode == "decode":
        out = ep.decode_layer(be, part, dev(a), wr, local, shp.k, bias=None if bias is None else dev(bias))
    else:
        out = ep.prefill_layer(be, part, dev(a), wr, local, shp.k)
    torch.cuda.synchronize()
    o = host(out)
    assert_close(o, ref["out"], what=f"{mode} out")
    assert_close(o - a, ref["out"] - a, what=f"{mode} moe delta")

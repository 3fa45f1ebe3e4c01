"""The benchmark's multi-rank plumbing on CPU: two gloo ranks, as under
torchrun with --gpus 2 (replicas: the per-rank device times are reduced to
their maximum, the whole-job rate is all ranks' units over that time, and the
CPU reference arm runs on rank 0 only)."""
import json
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    import bench
    r, w, local = bench.dist_env()
    dist = bench.init_dist(w, "gloo")
    elapsed_ms = [3.0, 5.0][rank]          # this rank's device time
    mx = bench.max_over_ranks(elapsed_ms, w)
    rate = bench.aggregate_rate(units_per_rank=4 * 100, world=w, seconds_max=mx / 1e3)
    dist.barrier()
    with open(os.path.join(out_dir, f"rank{r}.json"), "w") as f:
        json.dump({"rank": r, "world": w, "local": local, "max_ms": mx, "rate": rate}, f)
    dist.destroy_process_group()


def test_two_gloo_ranks_reduce_to_the_slowest(tmp_path):
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, d in enumerate(res):
        assert d["rank"] == r and d["world"] == 2 and d["local"] == r
        assert d["max_ms"] == 5.0                      # every rank sees the slowest rank's time
        assert d["rate"] == pytest.approx(2 * 400 / 5e-3)   # all ranks' units over that time


def test_reference_arm_runs_on_rank_zero_only():
    sys.path.insert(0, ROOT)
    import argparse
    import bench
    args = argparse.Namespace(workload="verify_b1", steps=1, warmup=3)
    assert bench.run_reference(args, rank=1, world=2) is None

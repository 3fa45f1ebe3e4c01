"""Host-side logic of bench.py that needs no GPU: the stored DRAM traffic of
the dominant kernels (profiles/traffic.json) is reported only while every
source file of the profiled kernel is unchanged, and the roofline peaks come
from MEASURED_PEAKS.json."""
import json
import os
import shutil
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

CSRC = os.path.join(ROOT, "speculative_decoding_verification_router_b200", "csrc")


def _traffic():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        return json.load(f)


def test_traffic_entries_name_existing_sources_and_captures():
    d = _traffic()
    assert d, "no stored traffic"
    for key, e in d.items():
        kernel, workload = key.split(":")
        assert kernel in ("moe_stream_layer", "gemm1_stream", "gemm2_stream", "gemm1_tiled", "gemm2_tiled")
        names = e.get("sources") or [e["source"]]
        for n in names:
            assert os.path.exists(os.path.join(CSRC, n)), (key, n)
        assert os.path.exists(os.path.join(ROOT, e["capture"])), (key, e["capture"])
        assert e["bytes_per_launch"] > 0


def test_traffic_is_reported_only_for_unchanged_sources(tmp_path, monkeypatch):
    key, e = next(iter(_traffic().items()))
    kernel, workload = key.split(":")
    names = e.get("sources") or [e["source"]]
    # a private copy of the tree that bench reads: profiles + the kernel's sources
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "speculative_decoding_verification_router_b200" / "csrc"
    csrc.mkdir(parents=True)
    for n in names:
        shutil.copy(os.path.join(CSRC, n), csrc / n)
    entry = dict(e, source_sha=bench.sources_sha(names))
    (root / "profiles" / "traffic.json").write_text(json.dumps({key: entry}))
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.traffic_from_profile(kernel, workload) == e["bytes_per_launch"]
    assert bench.traffic_from_profile(kernel, "another_workload") is None
    # any change to any of the kernel's files makes the stored figure stale
    with open(csrc / names[-1], "a") as f:
        f.write("\n// changed\n")
    assert bench.traffic_from_profile(kernel, workload) is None
    # a missing source file also reads as stale, not as an error
    os.remove(csrc / names[-1])
    assert bench.traffic_from_profile(kernel, workload) is None


def test_peaks_come_from_the_measured_file():
    p = bench.load_peaks()
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        assert p["source"] == "measured"
        assert p["hbm_gbs"] == d["hbm_gbs"] and p["bf16_tflops"] == d["bf16_tflops"]
        assert p["bf16_tflops_sustained"] == d.get("bf16_tflops_sustained", d["bf16_tflops"])
    else:
        assert p["source"] == "fallback"

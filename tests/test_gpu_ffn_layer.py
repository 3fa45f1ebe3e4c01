"""GPU parity of moe_expert_ffn, the whole layer and the vocab head.

Expert outputs and layer outputs: max |gpu - ref| / max |ref| <= 2e-2 and
mean |gpu - ref| <= 2e-3 against the fp32 oracle (the GPU rounds the SwiGLU
activation h to bf16 and, on the tiled path, y_perm too).  Routing and the
permutation inside the layer are bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import assert_close, dev, host
from tests.inputs import routed_layer_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ms():
    from speculative_decoding_verification_router_b200 import moespec
    return moespec


def _weights_dev(lw):
    """Expert weights on the device in the packed layout the GEMMs read."""
    from speculative_decoding_verification_router_b200 import moespec as ms
    pk = lambda a: None if a is None else ms.pack_weights(dev(a))
    return pk(lw.w_gate_up), pk(lw.w_down), pk(lw.ws_gate_up), pk(lw.ws_down)


def _ffn_case(ms, shp, seed, y_dtype=torch.float32):
    a, lw, bias = routed_layer_inputs(shp, seed)
    ref = oracle.moe_layer(a, lw, shp.k, bias)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    off = dev(ref["offsets"])
    perm = dev(ref["perm"])
    y, ysh = ms.expert_ffn(dev(ref["xhat_bf16"]), off, perm, wgu, wd, wsgu, wsd, shp.k, y_dtype=y_dtype)
    torch.cuda.synchronize()
    return ref, host(y), (host(ysh) if ysh is not None else None)


FFN = [synth.TINY, synth.VERIFY_B1, synth.VERIFY_B32]


@pytest.mark.parametrize("shp", FFN, ids=[w.name for w in FFN])
def test_expert_ffn_streaming_parity(ms, shp):
    ref, y, ysh = _ffn_case(ms, shp, seed=0)
    assert_close(y, ref["y_perm"], what="y_perm")
    assert_close(ysh, ref["y_shared"], what="y_shared")


def test_expert_ffn_is_deterministic(ms):
    shp = synth.VERIFY_B32
    a, lw, bias = routed_layer_inputs(shp, 0)
    ref = oracle.moe_layer(a, lw, shp.k, bias)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    args = (dev(ref["xhat_bf16"]), dev(ref["offsets"]), dev(ref["perm"]), wgu, wd, wsgu, wsd, shp.k)
    y1, s1 = ms.expert_ffn(*args)
    y2, s2 = ms.expert_ffn(*args)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(s1, s2)


def test_expert_ffn_flags_oversized_group(ms):
    # offsets that give one expert more than T rows (a token routed to it
    # twice) are rejected on the device: the group is skipped and flagged,
    # the other groups and the shared expert are still computed
    shp = synth.TINY
    T, k, E = shp.T, shp.k, shp.E
    lw = synth.layer_weights(shp, 0)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    xb = synth.normal_bf16(0, "oversized_group_x", (T, shp.H), 1.0)
    off = np.full(E + 1, T * k, np.int32)
    off[0] = 0
    perm = (np.arange(T * k) % T).astype(np.int32)
    ws = ms.Workspace(ms.expert_ffn_workspace_size(T, shp.H, E, shp.I, shp.S, k))
    y, ysh = ms.expert_ffn(dev(xb), dev(off), dev(perm), wgu, wd, wsgu, wsd, k, ws=ws)
    assert ms.device_status(ws) == -6
    rs = oracle.expert_ffn_shared(oracle.widen_bf16(xb), lw.ws_gate_up, lw.ws_down)
    assert_close(host(ysh), rs, what="y_shared beside a rejected group")


@pytest.mark.parametrize("pattern", ["head_heavy", "one_full_expert"])
def test_expert_ffn_unequal_group_sizes(ms, pattern):
    # 128 tokens whose experts receive very different token counts.  The
    # streaming schedule cuts its split ranges at equal data cost (weights
    # plus 16-row token boxes), so a range over a 128-token group holds fewer
    # k-steps than one over a 2-token group; the results must not depend on it.
    shp = synth.VERIFY_B32
    T, k, E = shp.T, shp.k, shp.E
    lw = synth.layer_weights(shp, 3)
    rng = synth.stream(3, f"unequal_groups_{pattern}")
    if pattern == "head_heavy":
        p = (E - np.arange(E, dtype=np.float64)) ** 4
        idx = np.stack([rng.choice(E, k, replace=False, p=p / p.sum()) for _ in range(T)])
    else:
        # expert 0 in every token's set, the other five drawn uniformly
        idx = np.stack([np.concatenate([[0], 1 + rng.choice(E - 1, k - 1, replace=False)]) for _ in range(T)])
    idx = idx.astype(np.int32)
    off, perm, _ = oracle.permute(idx, E)
    counts = np.diff(off)
    assert counts.max() >= 48 and counts[counts > 0].min() <= 4   # the spread the case is about
    xb = synth.normal_bf16(3, f"unequal_groups_x_{pattern}", (T, shp.H), 1.0)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    y, ysh = ms.expert_ffn(dev(xb), dev(off), dev(perm), wgu, wd, wsgu, wsd, k)
    torch.cuda.synchronize()
    xw = oracle.widen_bf16(xb)
    assert_close(host(y), oracle.expert_ffn_routed(xw, lw.w_gate_up, lw.w_down, off, perm, k), what="y_perm")
    assert_close(host(ysh), oracle.expert_ffn_shared(xw, lw.ws_gate_up, lw.ws_down), what="y_shared")


@pytest.mark.parametrize("T", [129, 300])
def test_expert_ffn_tiled_ragged(ms, T):
    # the tiled (large-T) schedule on small shapes, with a ragged last tile
    shp = synth.MoEShape(f"tiled{T}", B=1, K=0, H=256, E=8, I=128, k=2, S=2, V=1024,
                         router_std=0.05, tokens=T)
    ref, y, ysh = _ffn_case(ms, shp, seed=1, y_dtype=torch.bfloat16)
    assert_close(y, ref["y_perm"], what="y_perm")
    assert_close(ysh, ref["y_shared"], what="y_shared")


def test_expert_ffn_tiled_flags_bad_token_index(ms):
    # the prefill-sized path gathers the token rows through bulk copies:
    # permutation entries outside [0, T) are flagged on the device and read
    # nothing outside x; every other row is computed as usual
    T = 300
    shp = synth.MoEShape("tiled_badidx", B=1, K=0, H=256, E=8, I=128, k=2, S=2, V=1024, router_std=0.05, tokens=T)
    ref, _, _ = _ffn_case(ms, shp, seed=4, y_dtype=torch.bfloat16)
    lw = synth.layer_weights(shp, 4)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    bad_rows = [5, 11, T * shp.k - 1]
    perm = ref["perm"].copy()
    perm[bad_rows] = [T + 7, -3, 1 << 30]
    ws = ms.Workspace(ms.expert_ffn_workspace_size(T, shp.H, shp.E, shp.I, shp.S, shp.k))
    y, ysh = ms.expert_ffn(dev(ref["xhat_bf16"]), dev(ref["offsets"]), dev(perm), wgu, wd, wsgu, wsd, shp.k,
                           y_dtype=torch.bfloat16, ws=ws)
    assert ms.device_status(ws) == -6
    keep = np.setdiff1d(np.arange(T * shp.k), bad_rows)
    assert_close(host(y)[keep], ref["y_perm"][keep], what="y_perm rows with valid tokens")
    assert_close(host(ysh), ref["y_shared"], what="y_shared")


def test_expert_ffn_prefill_sampled(ms):
    # full prefill size in the launch configuration the benchmark times;
    # the oracle recomputes a sample of rows and tokens one by one
    shp = synth.PREFILL
    a, lw, bias = routed_layer_inputs(shp, 0)
    xf, xb = oracle.rmsnorm(a)
    x = oracle.widen_bf16(xb)
    idx, w, _, _ = oracle.route_topk(x, lw.w_router, bias, shp.k)
    off, perm, slot = oracle.permute(idx, shp.E)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    y, ysh = ms.expert_ffn(dev(xb), dev(off), dev(perm), wgu, wd, wsgu, wsd, shp.k, y_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    g = np.random.default_rng(5)
    rows = np.unique(np.concatenate([g.choice(shp.T * shp.k, 96, replace=False), off[1:-1] - 1, off[:-1]]))
    rows = rows[(rows >= 0) & (rows < shp.T * shp.k)][:256]
    toks = np.unique(np.concatenate([g.choice(shp.T, 48, replace=False), [0, shp.T - 1]]))
    ry = oracle.expert_ffn_routed(x, lw.w_gate_up, lw.w_down, off, perm, shp.k, rows=rows)
    rs = oracle.expert_ffn_shared(x, lw.ws_gate_up, lw.ws_down, tokens=toks)
    yh = host(y[torch.from_numpy(rows).cuda().long()])
    sh = host(ysh[torch.from_numpy(toks).cuda().long()])
    assert_close(yh, ry[rows], what="y_perm rows")
    assert_close(sh, rs[toks], what="y_shared tokens")
    # rows the oracle did not recompute are still finite and of the right scale
    assert torch.isfinite(y.float()).all()


LAYER = [synth.TINY, synth.VERIFY_B1, synth.VERIFY_B32]


@pytest.mark.parametrize("shp", LAYER, ids=[w.name for w in LAYER])
def test_layer_parity_through_the_five_calls(ms, shp):
    a, lw, bias = routed_layer_inputs(shp, 0)
    ref = oracle.moe_layer(a, lw, shp.k, bias)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    ad = dev(a)
    xh = ms.rmsnorm(ad)
    idx, w = ms.route_topk(xh, dev(lw.w_router), None if bias is None else dev(bias), shp.k)
    off, perm, slot = ms.permute(idx, shp.E)
    y, ysh = ms.expert_ffn(xh, off, perm, wgu, wd, wsgu, wsd, shp.k)
    out = ms.combine(y, ysh, slot, w, ad)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(idx), ref["idx"])
    np.testing.assert_array_equal(host(off), ref["offsets"])
    np.testing.assert_array_equal(host(perm), ref["perm"])
    np.testing.assert_array_equal(host(slot), ref["slot"])
    o = host(out)
    assert_close(o, ref["out"], what="out")
    assert_close(o - a, ref["out"] - a, what="moe delta")


@pytest.mark.parametrize("shp", LAYER + [synth.MoEShape("tiled_layer", B=1, K=0, H=256, E=8, I=128, k=2, S=1,
                                                         V=1024, router_std=0.05, tokens=515)],
                         ids=[w.name for w in LAYER] + ["tiled_layer_t515"])
def test_layer_forward_composite(ms, shp):
    a, lw, bias = routed_layer_inputs(shp, 0)
    ref = oracle.moe_layer(a, lw, shp.k, bias)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    ws = ms.Workspace(ms.layer_workspace_size(shp.T, shp.H, shp.E, shp.I, shp.S, shp.k))
    out = ms.layer_forward(dev(a), dev(lw.w_router), None if bias is None else dev(bias), wgu, wd, wsgu, wsd,
                           shp.k, ws=ws)
    assert ms.device_status(ws) == 0
    o = host(out)
    assert_close(o, ref["out"], what="out")
    assert_close(o - a, ref["out"] - a, what="moe delta")


def test_tiny_fp32_weight_variant(ms):
    # fp32 variant of the tiny case: the oracle runs on the unrounded fp32
    # weights, the GPU on their bf16 rounding; the tolerance still holds
    shp = synth.TINY
    a, lw32, bias = routed_layer_inputs(shp, 0, weight_dtype="f32")
    lwb = synth.layer_weights(shp, 0, 0, "bf16")
    ref = oracle.moe_layer(a, lw32, shp.k, bias)
    wgu, wd, wsgu, wsd = _weights_dev(lwb)
    out = ms.layer_forward(dev(a), dev(lwb.w_router), None, wgu, wd, wsgu, wsd, shp.k)
    o = host(out)
    assert_close(o - a, ref["out"] - a, what="moe delta (fp32 weights)")


@pytest.mark.parametrize("T,V", [(4, 1024), (16, 1024), (128, 129280), (130, 2048)])
def test_lm_head_parity(ms, T, V):
    H = 1280 if V > 2048 else 256
    x = synth.normal_bf16(0, f"lmx{T}", (T, H), 1.0)
    wl = synth.normal_bf16(0, f"lmw{V}", (V, H), 0.02)
    out = ms.lm_head(dev(x), ms.pack_weights(dev(wl)))
    torch.cuda.synchronize()
    if V <= 2048:
        ref = oracle.lm_head(oracle.widen_bf16(x), wl)
        got = host(out)
    else:
        cols = np.random.default_rng(1).choice(V, 512, replace=False)
        cols = np.unique(np.concatenate([cols, [0, V - 1, 128, 129279 - 128]]))
        ref = oracle.lm_head(oracle.widen_bf16(x), wl[cols])
        got = host(out)[:, cols]
    # logits are written in bf16: one bf16 rounding of a ~N(0, 0.5) value
    assert_close(got, ref, max_rel=1e-2, mae=2e-3, what="logits")


@pytest.mark.parametrize("n,rows,cols", [(3, 256, 128), (1, 128, 64), (2, 1792, 1280), (1, 384, 896)])
def test_pack_weights_is_the_tile_permutation(ms, n, rows, cols):
    w = synth.normal_bf16(0, f"pack{n}x{rows}x{cols}", (n, rows, cols), 1.0)
    got = ms.bf16_to_bits(ms.pack_weights(dev(w))).reshape(-1)
    ref = w.reshape(n, rows // 128, 128, cols // 64, 64).transpose(0, 1, 3, 2, 4).reshape(-1)
    np.testing.assert_array_equal(got, ref)


def test_bounded_wait_reports_timeout(ms):
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    status = torch.full((1,), 7, dtype=torch.int32, device="cuda")
    old = ms.get_wait_limit_ns()
    try:
        ms.set_wait_limit_ns(2_000_000)          # 2 ms; nothing ever sets the flag
        ms.debug_bounded_wait(flag, 1, status)
        torch.cuda.synchronize()
        assert int(status.item()) == -5
        flag.fill_(1)
        ms.debug_bounded_wait(flag, 1, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
    finally:
        ms.set_wait_limit_ns(old)
    # the context is still usable afterwards
    assert torch.ones(4, device="cuda").sum().item() == 4


def test_trace_records_kernels(ms):
    shp = synth.VERIFY_B1
    a, lw, bias = routed_layer_inputs(shp, 0)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    ad, wr = dev(a), dev(lw.w_router)
    ms.trace_enable(64)
    try:
        ms.layer_forward(ad, wr, None, wgu, wd, wsgu, wsd, shp.k)
        torch.cuda.synchronize()
        recs = ms.trace_records()
    finally:
        ms.trace_disable()
        ms.trace_reset()
    names = [n for n, _ in recs]
    # a layer of at most 16 tokens is one persistent launch (routing, both GEMMs, their sums, combine)
    assert names == ["moe_stream_layer"], names
    # more tokens: the chain of launches
    shp32 = synth.VERIFY_B32
    a32, lw32, b32 = routed_layer_inputs(shp32, 0)
    w32 = _weights_dev(lw32)
    ms.trace_enable(64)
    try:
        ms.layer_forward(dev(a32), dev(lw32.w_router), dev(b32), *w32, shp32.k)
        torch.cuda.synchronize()
        names32 = [n for n, _ in ms.trace_records()]
    finally:
        ms.trace_disable()
        ms.trace_reset()
    assert names32 == ["route_cluster", "permute_scatter", "ffn_prep", "gemm1_stream", "ffn_finish", "gemm2_stream",
                       "ffn_finish", "combine"], names32
    assert all(t > 0 for _, t in recs)


def test_captured_step_replays_the_layer(ms):
    # a layer call captured once (with its input copy) and replayed equals a direct call
    shp = synth.VERIFY_B1
    a, lw, bias = routed_layer_inputs(shp, 3)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    wr = dev(lw.w_router)
    ws = ms.Workspace(ms.layer_workspace_size(shp.T, shp.H, shp.E, shp.I, shp.S, shp.k))
    a_h = torch.from_numpy(a).pin_memory()
    a_d = torch.empty_like(a_h, device="cuda")
    out = torch.empty_like(a_d)

    def fn():
        a_d.copy_(a_h, non_blocking=True)
        ms.layer_forward(a_d, wr, None, wgu, wd, wsgu, wsd, shp.k, ws=ws, out=out)

    step = ms.CapturedStep(fn)
    out.zero_()
    step()
    torch.cuda.synchronize()
    got = out.clone()
    direct = ms.layer_forward(dev(a), wr, None, wgu, wd, wsgu, wsd, shp.k)
    torch.cuda.synchronize()
    assert torch.equal(got, direct)


DEGENERATE = [
    synth.MoEShape("all_experts_k_eq_E", B=4, K=3, H=256, E=8, I=128, k=8, S=1, V=1024, router_std=0.05),
    synth.MoEShape("no_shared_expert", B=4, K=3, H=256, E=8, I=128, k=2, S=0, V=1024, router_std=0.05),
    synth.MoEShape("dense_one_expert", B=4, K=3, H=256, E=1, I=256, k=1, S=0, V=1024, router_std=0.05),
    synth.MoEShape("single_token", B=1, K=0, H=256, E=8, I=128, k=2, S=1, V=1024, router_std=0.05, tokens=1),
    synth.MoEShape("max_streaming_tokens", B=1, K=0, H=256, E=16, I=128, k=4, S=1, V=1024, router_std=0.05,
                   tokens=128),
]


@pytest.mark.parametrize("shp", DEGENERATE, ids=[w.name for w in DEGENERATE])
def test_layer_degenerate_shapes(ms, shp):
    # every expert chosen (k = E), no shared expert, a dense layer (E = 1), a
    # single token, and the largest batch of the streaming schedule
    a, lw, bias = routed_layer_inputs(shp, 0)
    ref = oracle.moe_layer(a, lw, shp.k, bias)
    wgu, wd, wsgu, wsd = _weights_dev(lw)
    ws = ms.Workspace(ms.layer_workspace_size(shp.T, shp.H, shp.E, shp.I, shp.S, shp.k))
    out = ms.layer_forward(dev(a), dev(lw.w_router), None if bias is None else dev(bias), wgu, wd, wsgu, wsd,
                           shp.k, ws=ws)
    assert ms.device_status(ws) == 0
    o = host(out)
    assert_close(o, ref["out"], what="out")
    assert_close(o - a, ref["out"] - a, what="moe delta")

"""GPU parity of moe_rmsnorm, moe_route_topk, moe_permute and moe_combine.

Indices and the permutation are compared bit for bit (inputs drawn so that
every token's top k+1 router logits are more than 1e-3 apart); gate weights
to a relative 1e-5 (expf vs the oracle's exp); RMSNorm outputs to one bf16
ulp; combine to fp32 rounding."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import dev, host
from tests.inputs import routed_xhat_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ms():
    from speculative_decoding_verification_router_b200 import moespec
    return moespec


@pytest.mark.parametrize("T,H", [(16, 256), (4, 1280), (128, 1280), (37, 1280), (1, 128)])
def test_rmsnorm_parity(ms, T, H):
    a = synth.normal(0, f"rms{T}", (T, H))
    xg = ms.rmsnorm(dev(a))
    torch.cuda.synchronize()
    xf, xb = oracle.rmsnorm(a)
    got = host(xg)
    ref = oracle.widen_bf16(xb)
    ulp = np.abs(ref) * 2.0 ** -7 + 1e-30
    assert np.all(np.abs(got - ref) <= ulp)
    assert np.mean(got == ref) > 0.99


WORK = [synth.TINY, synth.VERIFY_B1, synth.VERIFY_B32, synth.PREFILL]


@pytest.mark.parametrize("shp", WORK, ids=[w.name for w in WORK])
def test_route_parity(ms, shp):
    xb, wr, bias = routed_xhat_inputs(shp, seed=0)
    idx, w = ms.route_topk(dev(xb), dev(wr), None if bias is None else dev(bias), shp.k)
    torch.cuda.synchronize()
    ridx, rw, _, _ = oracle.route_topk(oracle.widen_bf16(xb), wr, bias, shp.k)
    np.testing.assert_array_equal(host(idx), ridx)
    np.testing.assert_allclose(host(w), rw, rtol=1e-5, atol=1e-7)
    # renormalised gates sum to one
    idx2, w2 = ms.route_topk(dev(xb), dev(wr), None if bias is None else dev(bias), shp.k, renormalize=True)
    np.testing.assert_array_equal(host(idx2), ridx)
    np.testing.assert_allclose(host(w2).astype(np.float64).sum(1), 1.0, atol=1e-5)


TC = [synth.MoEShape("tiny_e16", B=4, K=3, H=256, E=16, I=128, k=2, S=1, V=1024, router_std=0.05),
      synth.VERIFY_B32, synth.PREFILL,
      synth.MoEShape("ragged_tiles", B=1, K=0, H=1280, E=64, I=896, k=6, S=2, V=1024, router_std=0.05, tokens=1300)]


@pytest.mark.parametrize("shp", TC, ids=[w.name for w in TC])
def test_route_tensor_parity(ms, shp):
    # the router on the tensor cores (three bf16 parts of W_r, fp32 accumulation):
    # the same indices bit for bit, gates to fp32 rounding, with and without bias
    xb, wr, bias = routed_xhat_inputs(shp, seed=0)
    idx, w = ms.route_topk_tensor(dev(xb), dev(wr), None if bias is None else dev(bias), shp.k)
    torch.cuda.synchronize()
    ridx, rw, _, _ = oracle.route_topk(oracle.widen_bf16(xb), wr, bias, shp.k)
    np.testing.assert_array_equal(host(idx), ridx)
    np.testing.assert_allclose(host(w), rw, rtol=1e-5, atol=1e-7)
    idx2, w2 = ms.route_topk_tensor(dev(xb), dev(wr), None if bias is None else dev(bias), shp.k, renormalize=True)
    np.testing.assert_array_equal(host(idx2), ridx)
    np.testing.assert_allclose(host(w2).astype(np.float64).sum(1), 1.0, atol=1e-5)


def test_route_tensor_ties_go_to_the_lower_expert(ms):
    # equal router rows give equal logits: the lower expert is taken first
    T, H, E, k = 200, 256, 16, 4
    xb = synth.normal_bf16(4, "tc_ties_x", (T, H), 1.0)
    wr = synth.normal(4, "tc_ties_w", (E, H), 0.05)
    wr[9] = wr[2]
    wr[12] = wr[2]
    wr[5] = wr[14]
    idx, w = ms.route_topk_tensor(dev(xb), dev(wr), None, k)
    torch.cuda.synchronize()
    ridx, _, z, _ = oracle.route_topk(oracle.widen_bf16(xb), wr, None, k)
    got = host(idx)
    # where the oracle's top-k has no near-ties other than the exact duplicates, the sets agree
    zs = -np.sort(-z.astype(np.float64), axis=1)[:, : k + 1]
    gaps = -np.diff(zs, axis=1)
    clear = np.all((gaps == 0) | (gaps > 1e-3), axis=1)
    np.testing.assert_array_equal(got[clear], ridx[clear])
    assert clear.sum() > T // 2
    for t in np.nonzero(clear)[0]:
        for a_, b_ in [(2, 9), (2, 12), (9, 12), (5, 14)]:
            row = list(got[t])
            if a_ in row and b_ in row:
                assert row.index(a_) < row.index(b_)


def _random_idx(T, k, E, seed, skew=None):
    g = np.random.default_rng(seed)
    p = None if skew is None else g.dirichlet(np.full(E, skew))
    return np.stack([g.choice(E, size=k, replace=False, p=p) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("T,k,E,skew", [(16, 2, 8, None), (4, 6, 64, None), (128, 6, 64, 0.3),
                                        (36992, 6, 64, None), (700, 6, 64, 0.05), (3, 1, 1, None),
                                        (5000, 8, 256, None)])
def test_permute_parity(ms, T, k, E, skew):
    idx = _random_idx(T, k, E, seed=T + E, skew=skew)
    off, perm, slot = ms.permute(dev(idx), E)
    torch.cuda.synchronize()
    roff, rperm, rslot = oracle.permute(idx, E)
    np.testing.assert_array_equal(host(off), roff)
    np.testing.assert_array_equal(host(perm), rperm)
    np.testing.assert_array_equal(host(slot), rslot)


def test_permute_all_to_one_expert(ms):
    T, k, E = 9000, 1, 64
    idx = np.full((T, k), 17, np.int32)
    off, perm, slot = ms.permute(dev(idx), E)
    roff, rperm, rslot = oracle.permute(idx, E)
    np.testing.assert_array_equal(host(off), roff)
    np.testing.assert_array_equal(host(perm), rperm)
    np.testing.assert_array_equal(host(slot), rslot)


@pytest.mark.parametrize("ydt", ["f32", "bf16"])
@pytest.mark.parametrize("T,H,k,S", [(16, 256, 2, 1), (128, 1280, 6, 2), (5, 128, 3, 0)])
def test_combine_parity(ms, ydt, T, H, k, S):
    g = np.random.default_rng(T * H)
    y = g.standard_normal((T * k, H)).astype(np.float32)
    if ydt == "bf16":
        yb = synth.to_bf16_bits(y)
        y = oracle.widen_bf16(yb)
        ydev = dev(yb)
    else:
        ydev = dev(y)
    ysh = g.standard_normal((T, H)).astype(np.float32) if S else None
    res = g.standard_normal((T, H)).astype(np.float32)
    w = g.random((T, k)).astype(np.float32)
    slot = g.permutation(T * k).reshape(T, k).astype(np.int32)
    ob = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    out = ms.combine(ydev, None if ysh is None else dev(ysh), dev(slot), dev(w), dev(res), out_bf16=ob)
    torch.cuda.synchronize()
    ref = oracle.combine(y, ysh, slot, w, res)
    np.testing.assert_allclose(host(out), ref, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(host(ob), ref, rtol=1e-2, atol=1e-2)

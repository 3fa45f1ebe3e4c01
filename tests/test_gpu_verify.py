"""GPU parity of spec_verify_greedy against the oracle (bit-exact).

Greedy verification: argmax per position (lowest index on ties), longest
accepted prefix, one verifier token committed (jina.ai, "Modèle et
entraînement"; clawpit.io, "Speculative decoding without accuracy loss")."""
import numpy as np
import pytest
import torch

import oracle
from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import dev, host
from tests.inputs import verify_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ms():
    from speculative_decoding_verification_router_b200 import moespec
    return moespec


def _check(ms, lg, d):
    am, cm, n = ms.verify_greedy(dev(lg), dev(d))
    torch.cuda.synchronize()
    ram, rcm, rn = oracle.verify_greedy(lg, d)
    np.testing.assert_array_equal(host(am), ram)
    np.testing.assert_array_equal(host(cm), rcm)
    np.testing.assert_array_equal(host(n), rn)
    assert np.all((rn >= 1) & (rn <= d.shape[1] + 1))
    return rn


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_verify_tiny(ms, dtype):
    lg, d = verify_inputs(synth.TINY, seed=0, dtype=dtype)
    _check(ms, lg, d)


@pytest.mark.parametrize("B", [1, 32])
def test_verify_full_vocab_bf16(ms, B):
    shp = synth.STEP_B32 if B == 32 else synth.VERIFY_B1
    lg, d = verify_inputs(shp, seed=1, dtype="bf16")
    rn = _check(ms, lg, d)
    assert rn.min() >= 1


@pytest.mark.parametrize("V,dtype", [(1027, "f32"), (1027, "bf16"), (7, "bf16"), (3000, "f32"), (1, "f32")])
def test_verify_ragged_vocab(ms, V, dtype):
    shp = synth.MoEShape("ragged", B=5, K=3, H=128, E=2, I=128, k=1, S=0, V=V, router_std=1.0)
    lg, d = verify_inputs(shp, seed=2, dtype=dtype, V=V)
    _check(ms, lg, d)


@pytest.mark.parametrize("K", [0, 1, 2, 8])   # K = 0: plain greedy decoding
def test_verify_depths(ms, K):
    shp = synth.MoEShape("depth", B=6, K=K, H=128, E=2, I=128, k=1, S=0, V=5000, router_std=1.0, p_match=0.8)
    lg, d = verify_inputs(shp, seed=3, dtype="bf16")
    _check(ms, lg, d)


def test_verify_ties_and_extremes(ms):
    g = np.random.default_rng(4)
    B, K, V = 8, 3, 4096
    lg = np.round(g.standard_normal((B, K + 1, V)) * 2).astype(np.float32)   # many exact ties
    lg[0, :, :] = 1.0                                                       # whole rows tied
    lg[1, :, -1] = 100.0                                                    # max at the last index
    am_true = np.stack([[int(np.argmax(lg[b, j])) for j in range(K + 1)] for b in range(B)])
    d = am_true[:, :K].astype(np.int32).copy()
    d[2, 0] += 1                          # first draft rejected
    d[3, 2] = (d[3, 2] + 1) % V           # third rejected
    _check(ms, lg, d)
    _check(ms, synth.to_bf16_bits(lg).reshape(lg.shape), d)
    # all accepted: bonus token committed, count K+1
    am, cm, n = ms.verify_greedy(dev(lg), dev(am_true[:, :K].astype(np.int32).copy()))
    assert np.all(host(n) == K + 1)
    np.testing.assert_array_equal(host(cm), am_true)

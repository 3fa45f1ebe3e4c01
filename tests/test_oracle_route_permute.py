"""Pins for the oracle's RMSNorm, router/top-k and permutation.

Each check compares the oracle with something other than itself: a library
routine (numpy sort/argsort/bincount, scipy softmax, fp64 matmul), a closed
form, an invariant, or brute force over all orderings on tiny inputs.
"""
import itertools

import numpy as np
import pytest
import scipy.special

import oracle
from speculative_decoding_verification_router_b200 import synth

pytestmark = pytest.mark.usefixtures("oracle_lib")


# ---------------------------------------------------------------- RMSNorm

def test_rmsnorm_constant_row_is_sign():
    # a = c * 1  ->  a / sqrt(c^2 + eps) ~= sign(c)
    a = np.array([[3.0] * 8, [-0.5] * 8], np.float32)
    xf, _ = oracle.rmsnorm(a, eps=0.0)
    np.testing.assert_allclose(xf, np.sign(a), rtol=1e-7)


def test_rmsnorm_unit_rms_and_scale_invariance():
    g = np.random.default_rng(1)
    a = g.standard_normal((5, 64)).astype(np.float32)
    xf, _ = oracle.rmsnorm(a, eps=0.0)
    np.testing.assert_allclose(np.sqrt((xf.astype(np.float64) ** 2).mean(1)), 1.0, rtol=1e-6)
    xf2, _ = oracle.rmsnorm(a * np.float32(4.0), eps=0.0)   # power of two: exact scaling
    np.testing.assert_allclose(xf2, xf, rtol=1e-6, atol=1e-7)


def test_rmsnorm_gain_and_eps():
    a = np.array([[1.0, -1.0, 1.0, -1.0]], np.float32)
    gamma = np.array([1.0, 2.0, 3.0, 4.0], np.float32)
    xf, _ = oracle.rmsnorm(a, gamma=gamma, eps=3.0)          # 1/sqrt(1+3) = 0.5
    np.testing.assert_allclose(xf[0], [0.5, -1.0, 1.5, -2.0], rtol=1e-7)


def test_bf16_rounding_matches_torch():
    torch = pytest.importorskip("torch")
    g = np.random.default_rng(2)
    x = (g.standard_normal(100000) * np.exp(g.uniform(-20, 20, 100000))).astype(np.float32)
    # exact halfway cases: tie to even
    x = np.concatenate([x, np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8], np.float32)])
    ours = oracle.bf16_round(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


# ---------------------------------------------------------------- router

def _brute_topk(z, k):
    # full sort by (value descending, index ascending): numpy lexsort
    T, E = z.shape
    out = np.empty((T, k), np.int64)
    for t in range(T):
        order = np.lexsort((np.arange(E), -z[t].astype(np.float64)))
        out[t] = order[:k]
    return out


@pytest.mark.parametrize("T,H,E,k", [(7, 16, 8, 2), (5, 32, 16, 6), (3, 8, 4, 4), (9, 24, 64, 6)])
def test_router_matches_library_sort_and_softmax(T, H, E, k):
    g = np.random.default_rng(T * 100 + E)
    x = g.standard_normal((T, H)).astype(np.float32)
    w = (g.standard_normal((E, H)) * 0.5).astype(np.float32)
    bias = g.standard_normal((T, E)).astype(np.float32)
    idx, wt, z, p = oracle.route_topk(x, w, bias, k)
    zref = (x.astype(np.float64) @ w.astype(np.float64).T).astype(np.float32) + bias
    np.testing.assert_allclose(z, zref, rtol=1e-6, atol=1e-6)
    np.testing.assert_array_equal(idx, _brute_topk(z, k))
    pref = scipy.special.softmax(z.astype(np.float64), axis=1)
    np.testing.assert_allclose(p, pref, rtol=1e-6, atol=1e-9)
    np.testing.assert_allclose(wt, np.take_along_axis(pref, idx.astype(np.int64), 1), rtol=1e-6)
    s = wt.astype(np.float64).sum(1)
    assert np.all(s <= 1 + 1e-6) and np.all(s >= k / E - 1e-6)
    np.testing.assert_allclose(p.astype(np.float64).sum(1), 1.0, atol=1e-6)


def test_router_brute_force_all_orderings_tiny():
    # E = 4: check the selected ordered tuple is the lexicographically best
    g = np.random.default_rng(5)
    for trial in range(50):
        z = np.round(g.standard_normal((1, 4)) * 2) / 2            # frequent exact ties
        x = np.eye(4, dtype=np.float32)[:1] * 0 + 1.0
        w = np.zeros((4, 4), np.float32)
        bias = z.astype(np.float32)
        for k in (1, 2, 3, 4):
            idx, *_ = oracle.route_topk(x, w, bias, k)
            best = None
            for perm in itertools.permutations(range(4), k):
                key = tuple((-bias[0, e], e) for e in perm)
                # a valid top-k order is sorted by (value desc, index asc) and
                # takes the k best under that order
                if best is None or key < best[0]:
                    best = (key, perm)
            assert tuple(idx[0]) == best[1], (trial, k, bias, idx)


def test_router_special_cases():
    g = np.random.default_rng(6)
    x = g.standard_normal((6, 16)).astype(np.float32)
    w = g.standard_normal((8, 16)).astype(np.float32)
    idx1, w1, z, p = oracle.route_topk(x, w, None, 1)
    np.testing.assert_array_equal(idx1[:, 0], np.argmax(z, axis=1))           # k = 1 is argmax
    np.testing.assert_allclose(w1[:, 0], p.max(1), rtol=1e-7)
    idx8, w8, z, p = oracle.route_topk(x, w, None, 8)                         # k = E: full order
    np.testing.assert_array_equal(idx8, np.argsort(-z, axis=1, kind="stable"))
    np.testing.assert_allclose(w8.astype(np.float64).sum(1), 1.0, atol=1e-6)


def test_router_ties_pick_lowest_index():
    x = np.ones((1, 4), np.float32)
    w = np.zeros((6, 4), np.float32)
    bias = np.array([[0.0, 1.0, 1.0, 0.5, 1.0, 0.5]], np.float32)
    idx, *_ = oracle.route_topk(x, w, bias, 5)
    assert list(idx[0]) == [1, 2, 4, 3, 5]


def test_router_renormalize_sums_to_one():
    g = np.random.default_rng(7)
    x = g.standard_normal((10, 32)).astype(np.float32)
    w = g.standard_normal((16, 32)).astype(np.float32)
    _, wt, _, p = oracle.route_topk(x, w, None, 3, renormalize=True)
    np.testing.assert_allclose(wt.astype(np.float64).sum(1), 1.0, atol=1e-6)
    _, wt0, _, _ = oracle.route_topk(x, w, None, 3, renormalize=False)
    np.testing.assert_allclose(wt / wt.sum(1, keepdims=True), wt0 / wt0.sum(1, keepdims=True), rtol=1e-6)


# ---------------------------------------------------------------- permute

@pytest.mark.parametrize("T,k,E", [(16, 2, 8), (4, 6, 64), (128, 6, 64), (1, 1, 1), (37, 3, 5)])
def test_permute_is_stable_grouping(T, k, E):
    g = np.random.default_rng(T + k + E)
    idx = np.stack([g.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    off, perm, slot = oracle.permute(idx, E)
    flat = idx.reshape(-1)
    # offsets: exclusive scan of the histogram (numpy bincount + cumsum)
    counts = np.bincount(flat, minlength=E)
    np.testing.assert_array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
    # order: a stable sort of the flattened pairs by expert (numpy argsort, stable)
    order = np.argsort(flat, kind="stable")
    np.testing.assert_array_equal(perm, order // k)
    # slot_of is the inverse map and a bijection onto 0..T*k-1
    np.testing.assert_array_equal(np.sort(slot.reshape(-1)), np.arange(T * k))
    np.testing.assert_array_equal(slot.reshape(-1)[order], np.arange(T * k))
    for t in range(T):
        for j in range(k):
            r = slot[t, j]
            assert perm[r] == t and off[idx[t, j]] <= r < off[idx[t, j] + 1]


def test_synth_router_inputs_have_clear_gaps_after_resampling():
    # the helper used by GPU tests keeps a >1e-3 gap among the top k+1 logits
    from tests.inputs import routed_layer_inputs
    shp = synth.TINY
    a, lw, bias = routed_layer_inputs(shp, seed=0)
    xf, xb = oracle.rmsnorm(a)
    _, _, z, _ = oracle.route_topk(oracle.widen_bf16(xb), lw.w_router, bias, shp.k)
    zs = -np.sort(-z.astype(np.float64), axis=1)[:, : shp.k + 1]
    assert np.all(np.diff(-zs, axis=1) > 1e-3)

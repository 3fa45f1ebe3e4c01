"""Pins for the oracle's greedy verify and the lossless property.

- hand-worked cases of the acceptance rule (tests/golden/verify_cases.json);
- argmax equals numpy.argmax (first maximal index) on random and tied rows;
- n_committed in 1..K+1, all-correct drafts give K+1, a wrong first draft 1;
- the mean of tau over many seeds matches the closed form sum_i p^i;
- speculative greedy decoding emits the same bytes as plain greedy decoding
  over 200 steps; a perfect drafter gives tau = K+1, a wrong one tau = 1.
"""
import json
import os

import numpy as np
import pytest

import oracle
from oracle import spec_decode as sd
from speculative_decoding_verification_router_b200 import synth, metrics

pytestmark = pytest.mark.usefixtures("oracle_lib")
GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _rows_with_argmax(am, V, rng):
    rows = rng.standard_normal((len(am), V)).astype(np.float32)
    for j, a in enumerate(am):
        rows[j, a] = rows[j].max() + 1.0
    return rows


def test_verify_golden_cases():
    doc = json.load(open(os.path.join(GOLD, "verify_cases.json")))
    V = doc["V"]
    rng = np.random.default_rng(0)
    for c in doc["cases"]:
        K = c["K"]
        lg = _rows_with_argmax(c["row_argmax"], V, rng)[None]
        am, cm, n = oracle.verify_greedy(lg, np.array([c["draft"]], np.int32))
        assert list(am[0]) == c["row_argmax"], c["name"]
        assert list(cm[0]) == c["committed"], c["name"]
        assert int(n[0]) == c["n_committed"], c["name"]
    for c in doc["tie_cases"]:
        lg = np.array([[c["row"], c["row"]]], np.float32)
        am, _, _ = oracle.verify_greedy(lg, np.zeros((1, 1), np.int32))
        assert am[0, 0] == c["argmax"], c["name"]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_verify_argmax_is_first_maximum(dtype):
    shp = synth.TINY
    lg = synth.logits(shp, seed=3, dtype=dtype)
    am, cm, n = oracle.verify_greedy(lg, np.zeros((shp.B, shp.K), np.int32))
    wide = oracle.widen_bf16(lg) if dtype == "bf16" else lg
    np.testing.assert_array_equal(am, np.argmax(wide, axis=2))
    assert np.all((n >= 1) & (n <= shp.K + 1))


def test_verify_bf16_ties_are_common_and_resolved_low():
    # vocab 129,280 bf16 N(0,1) rows: exact ties at the maximum do occur
    g = np.random.default_rng(4)
    z = synth.to_bf16_bits(g.standard_normal((64, 1, 4096)).astype(np.float32))
    wide = oracle.widen_bf16(z)
    am, _, _ = oracle.verify_greedy(np.concatenate([z, z], axis=1), np.zeros((64, 1), np.int32))
    np.testing.assert_array_equal(am[:, 0], np.argmax(wide[:, 0], axis=1))
    ties = sum(int((wide[b, 0] == wide[b, 0].max()).sum() > 1) for b in range(64))
    assert ties >= 1


def test_verify_invariants_random():
    g = np.random.default_rng(5)
    for trial in range(200):
        B, K, V = 3, int(g.integers(1, 8)), int(g.integers(2, 50))
        lg = g.standard_normal((B, K + 1, V)).astype(np.float32)
        am_true = np.argmax(lg, axis=2)
        # all drafts correct -> K+1 committed, equal to the argmax row
        am, cm, n = oracle.verify_greedy(lg, am_true[:, :K].astype(np.int32))
        assert np.all(n == K + 1)
        np.testing.assert_array_equal(cm, am_true)
        # first draft wrong -> exactly one token, the verifier's own
        bad = ((am_true[:, :K] + 1) % V).astype(np.int32)
        am, cm, n = oracle.verify_greedy(lg, bad)
        assert np.all(n == 1)
        np.testing.assert_array_equal(cm[:, 0], am_true[:, 0])
        assert np.all(cm[:, 1:] == -1)
        # random drafts: committed prefix equals the argmax prefix; count in range
        d = g.integers(0, V, (B, K)).astype(np.int32)
        am, cm, n = oracle.verify_greedy(lg, d)
        assert np.all((n >= 1) & (n <= K + 1))
        for b in range(B):
            m = 0
            while m < K and d[b, m] == am_true[b, m]:
                m += 1
            assert n[b] == m + 1
            np.testing.assert_array_equal(cm[b, : m + 1], am_true[b, : m + 1])


def test_verify_without_drafts_is_greedy_decoding():
    # K = 0: one row per sequence, its argmax committed, one token per step
    g = np.random.default_rng(6)
    lg = g.standard_normal((5, 1, 300)).astype(np.float32)
    am, cm, n = oracle.verify_greedy(lg, np.zeros((5, 0), np.int32))
    np.testing.assert_array_equal(am[:, 0], np.argmax(lg[:, 0], axis=1))
    np.testing.assert_array_equal(cm, am)
    assert np.all(n == 1)


def test_mean_tau_matches_closed_form():
    # drafts match iid with p_eff = p + (1-p)/V; E[tau] = sum_{i<=K} p_eff^i
    shp = synth.TINY
    taus = []
    for seed in range(400):
        lg = synth.logits(shp, seed=seed, dtype="f32")
        am, _, _ = oracle.verify_greedy(lg, np.zeros((shp.B, shp.K), np.int32))
        d = synth.drafts(am[:, : shp.K], shp.p_match, shp.V, seed)
        _, _, n = oracle.verify_greedy(lg, d)
        taus.extend(n.tolist())
    taus = np.array(taus, np.float64)
    p_eff = shp.p_match + (1 - shp.p_match) / shp.V
    expect = metrics.expected_tau_iid(p_eff, shp.K)
    se = taus.std(ddof=1) / np.sqrt(len(taus))
    assert abs(taus.mean() - expect) < 4 * se, (taus.mean(), expect, se)


# ---------------------------------------------------------------- lossless

PROMPT = [3, 17, 99, 200, 5, 42, 8, 130]


@pytest.fixture(scope="module")
def tiny_decoder():
    dec = sd.make_decoder(0)
    return dec, sd.greedy_decode(dec, PROMPT, 200)


@pytest.mark.parametrize("scale", [0.05, 0.2])
def test_speculative_equals_greedy_200_steps(tiny_decoder, scale):
    dec, greedy = tiny_decoder
    assert len(set(greedy)) >= 10          # the stream is not a trivial loop
    spec, taus = sd.speculative_decode(dec, sd.greedy_drafter(sd.perturbed(dec, scale, 1)),
                                       PROMPT, 200, K=3)
    assert bytes(spec) == bytes(greedy)
    assert all(1 <= t <= 4 for t in taus)
    assert 1.0 < np.mean(taus) < 4.0       # some, not all, drafts accepted


def test_perfect_and_wrong_drafters(tiny_decoder):
    dec, greedy = tiny_decoder
    spec, taus = sd.speculative_decode(dec, sd.greedy_drafter(dec), PROMPT, 60, K=3)
    assert bytes(spec) == bytes(greedy[:60]) and all(t == 4 for t in taus)
    spec, taus = sd.speculative_decode(dec, sd.wrong_drafter(dec), PROMPT, 40, K=3)
    assert bytes(spec) == bytes(greedy[:40]) and all(t == 1 for t in taus)


# ---------------------------------------------------------------- pages' numbers

def test_reporting_identities_against_printed_numbers():
    n = {k: v["value"] for k, v in json.load(open(os.path.join(GOLD, "pages_numbers.json"))).items()
         if isinstance(v, dict)}
    # acceptance rate quoted with tau: (2.73 - 1) / 3 = 57.67 % ~ 57.6 %
    assert abs(metrics.acceptance_rate(n["tau_k3_eager"], n["K"]) - n["acceptance_rate"]) < 1e-3
    # speedup 83.1 / 42.7 = 1.946 ~ 1.95
    assert abs(n["spec_eager_tok_s"] / n["ar_eager_tok_s"] - n["speedup_eager"]) < 5e-3
    # c = tau / S = 2.73 / 1.946 = 1.40
    c_e = metrics.step_cost(n["tau_k3_eager"], n["spec_eager_tok_s"] / n["ar_eager_tok_s"])
    assert abs(c_e - n["cost_eager_ar_steps"]) < 5e-3
    # overhead of a speculative step ~ 9 ms in both modes
    assert abs(metrics.spec_overhead_s(n["cost_eager_ar_steps"], n["ar_eager_tok_s"]) * 1e3
               - n["spec_overhead_ms"]) < 0.5
    assert abs(metrics.spec_overhead_s(n["cost_graphs_ar_steps"], n["ar_graphs_tok_s"]) * 1e3
               - n["spec_overhead_ms"]) < 0.6
    # K = 1 with graphs: 185.6 / 158.3 = 1.17
    assert abs(n["k1_graphs_tok_s"] / n["ar_graphs_tok_s"] - n["speedup_k1_graphs"]) < 5e-3
    # iid drafts at p = 0.576 would give tau = 2.099, not 2.73
    assert abs(metrics.expected_tau_iid(0.576, 3) - 2.0993) < 1e-3
    assert metrics.verified_tokens_per_s(32, 3, 1.0) == 128

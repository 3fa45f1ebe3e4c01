"""The precision argument of the tensor-core router, checked numerically on
the host (no GPU): fp32 router weights split into three bf16 terms
hi = bf16(w), mid = bf16(w - hi), lo = bf16(w - hi - mid) (each difference
taken in fp32, as the split kernel does) carry w to about 2^-24 relative;
every product of a bf16 activation with a bf16 term is exact in fp32; so a
dot product accumulated in fp32 over the three terms differs from the exact
(fp64) one by no more than fp32 accumulation of the same length does.  The
routing's tie margin (adjacent top-(k+1) logits at least 1e-3 apart in the
tests) is far above that difference, which is why the tensor-core router's
indices match the oracle's bit for bit."""
import numpy as np

from speculative_decoding_verification_router_b200 import synth


def _bf16(x):
    """Round fp32 values to bf16 (nearest, ties to even), back as fp32."""
    return synth.bf16_bits_to_f32(synth.to_bf16_bits(np.asarray(x, np.float32)))


def _split(w):
    w = np.asarray(w, np.float32)
    hi = _bf16(w)
    r1 = (w - hi).astype(np.float32)
    mid = _bf16(r1)
    r2 = (r1 - mid).astype(np.float32)
    return hi, mid, _bf16(r2)


def test_three_bf16_terms_carry_the_fp32_weight():
    rng = np.random.default_rng(7)
    w = (rng.standard_normal(200_000) / np.sqrt(1280)).astype(np.float32)
    w[:4] = [0.0, 1.0, -3.0e-8, 65504.0]   # zero, a power of two, a tiny and a large value
    hi, mid, lo = _split(w)
    rec = hi.astype(np.float64) + mid.astype(np.float64) + lo.astype(np.float64)
    err = np.abs(rec - w.astype(np.float64))
    assert np.all(err <= 2.0 ** -24 * np.abs(w.astype(np.float64)) + 1e-45)
    # one or two terms are not enough: the split is needed for fp32 fidelity
    assert np.max(np.abs(hi.astype(np.float64) + mid - w) / np.maximum(np.abs(w), 1e-30)) > 2.0 ** -20


def test_bf16_products_are_exact_in_fp32():
    rng = np.random.default_rng(8)
    x = _bf16(rng.standard_normal(100_000))
    for t in _split((rng.standard_normal(100_000) / 40).astype(np.float32)):
        p32 = (x * t).astype(np.float32)
        p64 = x.astype(np.float64) * t.astype(np.float64)
        np.testing.assert_array_equal(p32.astype(np.float64), p64)


def test_split_dot_products_stay_within_fp32_accumulation_error():
    H, E = 1280, 64
    rng = np.random.default_rng(9)
    wr = (rng.standard_normal((E, H)) / np.sqrt(H)).astype(np.float32)
    x = _bf16(rng.standard_normal((16, H)))
    hi, mid, lo = _split(wr)
    exact = x.astype(np.float64) @ wr.astype(np.float64).T
    # fp32 accumulation in k order over the three terms (one possible MMA order)
    acc = np.zeros((16, E), np.float32)
    for h in range(H):
        for t in (hi, mid, lo):
            acc = (acc + (x[:, h:h + 1] * t[:, h][None, :]).astype(np.float32)).astype(np.float32)
    bound = 3 * H * 2.0 ** -24 * (np.abs(x).astype(np.float64) @ np.abs(wr).astype(np.float64).T)
    assert np.all(np.abs(acc.astype(np.float64) - exact) <= bound)
    # and far below the 1e-3 gap the routing tests keep between adjacent top-(k+1) logits
    assert np.max(np.abs(acc - exact)) < 1e-4

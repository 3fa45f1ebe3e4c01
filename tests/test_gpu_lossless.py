"""The lossless property on the GPU path, with batch-invariant schedules.

The pages call FastMTP's greedy verification lossless: what it commits is
byte-identical to plain greedy decoding (the d9249 blog, "핵심 아이디어 / 구조
/ 동작 방식"; clawpit.io, "Speculative decoding without accuracy loss").  A
small decoder runs its MoE layers, final RMSNorm, vocabulary head and
verification through the library; the causal prefix-mean mixing that stands
in for attention is done on the host, per position in a fixed order (as in
the oracle's tiny decoder).  Plain greedy decoding feeds one position per
forward pass; speculative decoding feeds K+1 (the last committed token and K
drafts) and commits what spec_verify_greedy accepts.  With
ms_set_batch_invariant on, every committed token must come from logits that
are bit-identical to the greedy pass's for the same position, and the two
token streams must agree over 200 tokens."""
import numpy as np
import pytest
import torch

from speculative_decoding_verification_router_b200 import synth
from tests.gpu_util import dev, host

pytestmark = pytest.mark.gpu

V, H, L, E, I, K_TOP, S = 256, 128, 2, 8, 128, 2, 1
K = 3
PROMPT = [3, 17, 99, 200, 5, 42, 8, 130]
N_NEW = 200


@pytest.fixture(scope="module")
def ms():
    from speculative_decoding_verification_router_b200 import moespec
    return moespec


class GpuDecoder:
    """embedding -> L x [h + prefix_mean(h) -> MoE layer (library)] -> RMSNorm ->
    vocab head (library).  Keeps, per layer, the running fp32 sum of the layer
    inputs over the processed positions (the prefix mean's numerator)."""

    def __init__(self, ms, seed=0):
        self.ms = ms
        shp = synth.MoEShape("lossless", B=1, K=0, H=H, E=E, I=I, k=K_TOP, S=S, V=V, router_std=0.3,
                             weight_std=0.1, tokens=1)
        self.emb = synth.normal(seed, "lossless.emb", (V, H), 1.0)
        pk = lambda a: ms.pack_weights(dev(a))
        self.layers = []
        for l in range(L):
            lw = synth.layer_weights(shp, seed, l)
            self.layers.append((dev(lw.w_router), pk(lw.w_gate_up), pk(lw.w_down), pk(lw.ws_gate_up),
                                pk(lw.ws_down)))
        self.w_lm = pk(synth.normal_bf16(seed, "lossless.w_lm", (V, H), 0.5))
        self.cum = [np.zeros(H, np.float32) for _ in range(L)]   # sums over positions < self.n
        self.n = 0                                              # processed positions

    def snapshot(self):
        return [c.copy() for c in self.cum], self.n

    def restore(self, snap):
        self.cum, self.n = [c.copy() for c in snap[0]], snap[1]

    def forward(self, toks):
        """Logits [len(toks), V] (bf16 values) of the positions n .. n+len-1; advances n.
        Also returns, per position, the running sums after it (for rolling back)."""
        ms = self.ms
        h = self.emb[np.asarray(toks, np.int64)].astype(np.float32)
        T = h.shape[0]
        after = []
        for l, (wr, wgu, wd, wsgu, wsd) in enumerate(self.layers):
            u = np.empty_like(h)
            c = self.cum[l].copy()
            cums = []
            for j in range(T):
                c = (c + h[j]).astype(np.float32)
                cums.append(c.copy())
                u[j] = h[j] + (c / np.float32(self.n + j + 1)).astype(np.float32)
            after.append(cums)
            out = ms.layer_forward(dev(u), wr, None, wgu, wd, wsgu, wsd, K_TOP)
            torch.cuda.synchronize()
            h = host(out)
        xh = ms.rmsnorm(dev(h))
        lg = ms.lm_head(xh, self.w_lm)
        torch.cuda.synchronize()
        return lg, after

    def advance(self, after, keep):
        """Keep the first `keep` positions of the last forward pass."""
        if keep > 0:
            for l in range(L):
                self.cum[l] = after[l][keep - 1].copy()
        self.n += keep


def _greedy(ms, dec):
    dec.restore(dec.start)
    toks, rows = [PROMPT[-1]], []
    out = []
    while len(out) < N_NEW:
        lg, after = dec.forward([toks[-1]])
        dec.advance(after, 1)
        am, cm, n = ms.verify_greedy(lg.view(1, 1, V), torch.zeros((1, 0), dtype=torch.int32, device="cuda"))
        torch.cuda.synchronize()
        t = int(host(cm)[0, 0])
        rows.append(ms.bf16_to_bits(lg)[0].copy())
        out.append(t)
        toks.append(t)
    return out, rows


def _speculative(ms, dec, greedy_stream, seed=5):
    dec.restore(dec.start)
    g = np.random.default_rng(seed)
    last = PROMPT[-1]
    out, rows, taus = [], [], []
    while len(out) < N_NEW:
        pos = len(out)
        # drafts: the greedy continuation w.p. 0.7 per position, else a random token
        truth = greedy_stream[pos:pos + K] + [0] * max(0, pos + K - len(greedy_stream))
        d = [int(truth[i]) if g.random() < 0.7 else int(g.integers(0, V)) for i in range(K)]
        lg, after = dec.forward([last] + d)
        am, cm, n = ms.verify_greedy(lg.view(1, K + 1, V), dev(np.asarray([d], np.int32)))
        torch.cuda.synchronize()
        nc = int(host(n)[0])
        c = [int(x) for x in host(cm)[0, :nc]]
        bits = ms.bf16_to_bits(lg)
        rows += [bits[j].copy() for j in range(nc)]   # row j picked committed token j
        # positions of `last` and the accepted drafts were correct inputs: keep them
        dec.advance(after, nc)
        out += c
        taus.append(nc)
        last = c[-1]
    return out[:N_NEW], rows[:N_NEW], taus


def test_speculative_equals_greedy_on_the_gpu(ms):
    old = ms.get_batch_invariant()
    ms.set_batch_invariant(True)
    try:
        dec = GpuDecoder(ms)
        # the prompt's positions but the last, processed once; both runs start from here
        _, after = dec.forward(PROMPT[:-1])
        dec.advance(after, len(PROMPT) - 1)
        dec.start = dec.snapshot()
        greedy, grows = _greedy(ms, dec)
        spec, srows, taus = _speculative(ms, dec, greedy)
    finally:
        ms.set_batch_invariant(old)
    assert len(set(greedy)) >= 3   # the stream is not constant
    # every committed token was picked from the same bits as in greedy decoding
    for i in range(N_NEW):
        np.testing.assert_array_equal(srows[i], grows[i], err_msg=f"logits of position {i}")
    assert spec == greedy
    assert 1 < np.mean(taus) < K + 1 and min(taus) >= 1 and max(taus) <= K + 1


def test_batch_invariant_rows_do_not_depend_on_the_batch(ms):
    # the same token rows, alone and inside batches of other rows, through the
    # layer and the vocab head: bit-identical outputs with the setting on
    shp = synth.MoEShape("inv", B=1, K=0, H=1280, E=64, I=896, k=6, S=2, V=129280, router_std=0.05, tokens=1)
    lw = synth.layer_weights(shp, 3)
    pk = lambda a: ms.pack_weights(dev(a))
    wr, wgu, wd, wsgu, wsd = dev(lw.w_router), pk(lw.w_gate_up), pk(lw.w_down), pk(lw.ws_gate_up), pk(lw.ws_down)
    wl = pk(synth.normal_bf16(3, "inv.wlm", (4096, 1280), 0.02))
    rows = synth.normal(3, "inv.rows", (40, 1280), 1.0)
    old = ms.get_batch_invariant()
    ms.set_batch_invariant(True)
    try:
        outs, lgs = {}, {}
        for T in (1, 4, 16, 40):
            a = np.ascontiguousarray(rows[:T])
            o = ms.layer_forward(dev(a), wr, None, wgu, wd, wsgu, wsd, 6)
            xh = ms.rmsnorm(o)
            lg = ms.lm_head(xh, wl)
            torch.cuda.synchronize()
            outs[T], lgs[T] = host(o), ms.bf16_to_bits(lg)
    finally:
        ms.set_batch_invariant(old)
    for T in (4, 16, 40):
        np.testing.assert_array_equal(outs[T][:1], outs[1], err_msg=f"layer output, batch of {T}")
        np.testing.assert_array_equal(lgs[T][:1], lgs[1], err_msg=f"logits, batch of {T}")
    np.testing.assert_array_equal(outs[40][:16], outs[16])
    np.testing.assert_array_equal(lgs[40][:16], lgs[16])

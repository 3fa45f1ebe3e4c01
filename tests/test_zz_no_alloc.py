"""spec_verify_greedy_noalloc: greedy verification with no caller workspace.

It serves callers that cannot allocate device memory -- a plugin inside an
inference server whose memory belongs to the host application's pool, or a
real-time decode loop that may not call cudaMalloc once running.  Its scratch
is a static device array inside the library.  This file is collected last so
that a failure here does not hide the other GPU tests; it passes both on its
own in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from speculative_decoding_verification_router_b200 import synth

pytestmark = pytest.mark.gpu


def _noalloc():
    from speculative_decoding_verification_router_b200 import moespec as ms
    fn = ms.lib().spec_verify_greedy_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    fn.restype = I
    fn.argtypes = [P, I, P, I, I, I, P, P, P, P]
    return ms, fn


def _call(ms, fn, lg, d):
    B, K1, V = lg.shape
    am = torch.full((B, K1), -7, dtype=torch.int32, device="cuda")
    cm = torch.full((B, K1), -7, dtype=torch.int32, device="cuda")
    n = torch.full((B,), -7, dtype=torch.int32, device="cuda")
    st = fn(ctypes.c_void_p(lg.data_ptr()), 1 if lg.dtype == torch.bfloat16 else 0, ctypes.c_void_p(d.data_ptr()),
            B, K1 - 1, V, ctypes.c_void_p(am.data_ptr()), ctypes.c_void_p(cm.data_ptr()),
            ctypes.c_void_p(n.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st, am, cm, n


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_noalloc_matches_workspace_entry_point_on_two_calls(dtype):
    ms, fn = _noalloc()
    shapes = [synth.STEP_B32, synth.VERIFY_B1]          # two calls in a row, different batches
    for call, shp in enumerate(shapes):
        z = synth.logits(shp, seed=10 + call, dtype=dtype)
        lg = torch.from_numpy(z.view(np.int16)).view(torch.bfloat16).cuda() if dtype == "bf16" \
            else torch.from_numpy(z).cuda()
        # drafts: the verifier's own picks w.p. 0.6, taken from the workspace entry point
        am0, _, _ = ms.verify_greedy(lg, torch.zeros((shp.B, shp.K), dtype=torch.int32, device="cuda"))
        d = torch.from_numpy(synth.drafts(am0[:, : shp.K].cpu().numpy(), 0.6, shp.V, seed=call)).cuda()
        ref = ms.verify_greedy(lg, d)
        st, am, cm, n = _call(ms, fn, lg, d)
        torch.cuda.synchronize()
        assert st == 0, ms.STATUS.get(st, st)
        assert torch.equal(am, ref[0]) and torch.equal(cm, ref[1]) and torch.equal(n, ref[2])
        assert int(n.min()) >= 1 and int(n.max()) <= shp.K + 1


def test_noalloc_rejects_batches_beyond_its_static_scratch():
    ms, fn = _noalloc()
    B, K, V = 4097, 3, 16                                # 16,388 rows > 16,384
    lg = torch.zeros((B, K + 1, V), dtype=torch.bfloat16, device="cuda")
    d = torch.zeros((B, K), dtype=torch.int32, device="cuda")
    st, am, _, _ = _call(ms, fn, lg, d)
    torch.cuda.synchronize()
    assert st == -2                                      # MS_ERR_UNSUPPORTED, nothing launched
    assert int(am.min()) == -7 and int(am.max()) == -7

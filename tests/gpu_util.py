"""Helpers shared by the GPU parity tests (host <-> device, error metrics)."""
from __future__ import annotations

import numpy as np
import torch

from speculative_decoding_verification_router_b200 import synth

# Layer-output tolerance of the verify layer against the fp32 oracle:
# max |gpu - ref| / max |ref| <= 2e-2 and mean |gpu - ref| <= 2e-3.
MAX_REL = 2e-2
MAE = 2e-3


def dev(a: np.ndarray, dtype=None) -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()
    t = torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return t if dtype is None else t.to(dtype)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return synth.bf16_bits_to_f32(t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16))
    return t.contiguous().cpu().numpy()


def errs(gpu: np.ndarray, ref: np.ndarray):
    g = gpu.astype(np.float64)
    r = ref.astype(np.float64)
    d = np.abs(g - r)
    return float(d.max() / max(np.abs(r).max(), 1e-30)), float(d.mean())


def assert_close(gpu, ref, max_rel=MAX_REL, mae=MAE, what=""):
    mr, ma = errs(gpu, ref)
    assert mr <= max_rel and ma <= mae, f"{what}: max_rel={mr:.3e} (<= {max_rel}), mae={ma:.3e} (<= {mae})"
    return mr, ma

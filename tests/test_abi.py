"""C-ABI checks that need no GPU: the library loads, exports every function
include/moespec.h declares, and rejects bad arguments on the host before
launching anything."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moespec.h")
LIB = os.path.join(ROOT, "speculative_decoding_verification_router_b200", "libmoespec.so")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^\s*(?:MS_API\s+)?(?:const\s+)?[a-z_0-9]+\s*\**\s*([a-z_0-9]+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from speculative_decoding_verification_router_b200 import build
    build.build()
    return ctypes.CDLL(LIB)


def test_header_declares_the_hot_path_calls():
    names = _declared()
    for n in ["moe_route_topk", "moe_permute", "moe_expert_ffn", "moe_combine", "spec_verify_greedy",
              "moe_rmsnorm", "lm_head_logits", "moe_layer_forward"]:
        assert n in names
    assert len(names) >= 25


def test_library_exports_every_declared_symbol(lib):
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing


def test_host_validation_rejects_bad_arguments(lib):
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.moe_route_topk.restype = I
    lib.moe_route_topk.argtypes = [P, P, P, I, I, I, I, I, P, P, P]
    assert lib.moe_route_topk(None, None, None, 4, 1280, 64, 6, 0, None, None, None) == -1
    fake = P(4096)   # never dereferenced: validation fails first
    assert lib.moe_route_topk(fake, fake, None, 4, 1280, 64, 65, 0, fake, fake, None) == -1   # k > E
    assert lib.moe_route_topk(fake, fake, None, 4, 1000, 64, 6, 0, fake, fake, None) == -2   # H % 128
    lib.spec_verify_greedy.restype = I
    lib.spec_verify_greedy.argtypes = [P, I, P, I, I, I, P, P, P, P, ctypes.c_size_t, P]
    assert lib.spec_verify_greedy(fake, 1, fake, 2, 3, 100, fake, fake, fake, None, 0, None) == -3  # no ws
    assert lib.spec_verify_greedy(fake, 1, fake, 2, 9, 100, fake, fake, fake, fake, 1 << 20, None) == -2  # K > 8
    assert lib.spec_verify_greedy(fake, 7, fake, 2, 3, 100, fake, fake, fake, fake, 1 << 20, None) == -1  # dtype
    Z = ctypes.c_size_t
    lib.spec_verify_lm_head_greedy.restype = I
    lib.spec_verify_lm_head_greedy.argtypes = [P, P, P, I, I, I, I, P, P, P, P, Z, P]
    lib.spec_verify_lm_head_workspace_size.restype = Z
    lib.spec_verify_lm_head_workspace_size.argtypes = [I] * 4
    fused = lib.spec_verify_lm_head_greedy
    assert fused(None, fake, fake, 2, 3, 256, 1024, fake, fake, fake, fake, 1 << 30, None) == -1   # null xhat
    assert fused(fake, fake, fake, 2, 9, 256, 1024, fake, fake, fake, fake, 1 << 30, None) == -2   # K > 8
    assert fused(fake, fake, fake, 2, 3, 256, 1000, fake, fake, fake, fake, 1 << 30, None) == -2   # V % 128
    assert fused(fake, fake, fake, 2, 3, 256, 1024, fake, fake, fake, None, 0, None) == -3         # no ws
    assert lib.spec_verify_lm_head_workspace_size(32, 3, 1280, 129280) > 32 * 4 * 8
    assert lib.spec_verify_lm_head_workspace_size(0, 3, 1280, 129280) == 0
    # empty inputs are rejected before any launch
    lib.moe_permute.restype = I
    lib.moe_permute.argtypes = [P, I, I, I, P, P, P, P, Z, P]
    assert lib.moe_permute(fake, 0, 6, 64, fake, fake, fake, None, 0, None) == -1              # T = 0
    lib.moe_layer_forward.restype = I
    lib.moe_layer_forward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, Z, P]
    assert lib.moe_layer_forward(fake, fake, None, fake, fake, fake, fake, 0, 1280, 64, 896, 2, 6, 0, fake, fake,
                                 1 << 30, None) == -1                                          # T = 0
    assert lib.moe_layer_forward(fake, fake, None, fake, fake, fake, fake, 2048, 13312, 64, 896, 2, 6, 0, fake,
                                 fake, 1 << 40, None) == -2                                    # prefill H > 12288
    assert lib.spec_verify_greedy(fake, 1, fake, 0, 3, 100, fake, fake, fake, fake, 1 << 20, None) == -1  # B = 0
    assert lib.spec_verify_greedy(fake, 1, None, 2, 0, 100, fake, fake, fake, None, 0, None) == -3  # K = 0 needs no drafts
    lib.moe_expert_ffn_workspace_size.restype = ctypes.c_size_t
    lib.moe_expert_ffn_workspace_size.argtypes = [I] * 6
    assert lib.moe_expert_ffn_workspace_size(4, 1280, 64, 896, 2, 6) > 0
    assert lib.moe_expert_ffn_workspace_size(0, 1280, 64, 896, 2, 6) == 0
    lib.moe_rmsnorm.restype = I
    lib.moe_rmsnorm.argtypes = [P, P, I, I, ctypes.c_float, P, P]
    assert lib.moe_rmsnorm(fake, None, 4, 100, 1e-6, fake, None) == -2
    lib.ms_status_string.restype = ctypes.c_char_p
    lib.ms_status_string.argtypes = [I]
    assert lib.ms_status_string(-5) == b"device-side bounded wait timed out"


def test_binding_fails_loudly_without_library(tmp_path, monkeypatch):
    # the binding has no fallback: a missing library is an import error
    import importlib.util
    src = os.path.join(ROOT, "speculative_decoding_verification_router_b200", "moespec.py")
    dst = tmp_path / "moespec.py"
    dst.write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("moespec_copy", str(dst))
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError):
        spec.loader.exec_module(mod)


def test_product_path_never_imports_the_oracle():
    pkg = os.path.join(ROOT, "speculative_decoding_verification_router_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                txt = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in txt and "from oracle" not in txt, f
                assert "moe_oracle" not in txt, f


def test_batch_invariant_setting_round_trips(lib):
    # a host-side switch: no GPU needed to set and read it
    lib.ms_get_batch_invariant.restype = ctypes.c_int
    lib.ms_set_batch_invariant.argtypes = [ctypes.c_int]
    old = lib.ms_get_batch_invariant()
    try:
        lib.ms_set_batch_invariant(1)
        assert lib.ms_get_batch_invariant() == 1
        lib.ms_set_batch_invariant(0)
        assert lib.ms_get_batch_invariant() == 0
    finally:
        lib.ms_set_batch_invariant(old)

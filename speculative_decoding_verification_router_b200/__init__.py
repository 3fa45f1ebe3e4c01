"""MoE verify layer + greedy verification for B200 (sm_100a).

The compute lives in a C-ABI shared library (`libmoespec.so`, declared in
include/moespec.h); `moespec` is its thin ctypes binding.  Importing this
package loads nothing: `from speculative_decoding_verification_router_b200
import moespec` loads the library and fails loudly if it has not been built.
"""
__all__ = ["moespec", "synth", "metrics", "build"]

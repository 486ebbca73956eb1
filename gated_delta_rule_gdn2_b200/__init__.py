"""B200 (sm_100a) Gated DeltaNet-2 sequence mixer.

The computation lives in ``libgdn2.so`` (hand-written CUDA kernels behind the
C ABI of include/gdn2.h); this package is its ctypes binding.  The library is
loaded on first use, and every call fails loudly if it has not been built
(``python -m gated_delta_rule_gdn2_b200.build``): there is no other code path.
"""
from . import binding
from .binding import (GDN2_BF16, GDN2_FP32, LIB_PATH, STATUS, Gdn2Error, chunk_bwd, chunk_bwd_reduced,
                      chunk_fwd_gated, gdn2_debug_set, GDN2_DEBUG_WAIT_LIMIT, GDN2_DEBUG_WITHHOLD_READY,
                      chunk_bwd_varlen, chunk_fwd, chunk_fwd_reduced, chunk_fwd_varlen, decode_step,
                      decode_step_reduced, load, output_gate, output_gate_bwd, prologue, prologue_bwd)

# every C entry point, under its C name
for _name in binding.SIGNATURES:
    globals()[_name] = getattr(binding, _name)

__all__ = ["GDN2_BF16", "GDN2_FP32", "LIB_PATH", "STATUS", "Gdn2Error", "chunk_bwd", "chunk_bwd_reduced",
           "chunk_bwd_varlen", "chunk_fwd", "chunk_fwd_reduced", "chunk_fwd_varlen", "decode_step",
           "decode_step_reduced", "load", "chunk_fwd_gated", "GDN2_DEBUG_WAIT_LIMIT", "GDN2_DEBUG_WITHHOLD_READY",
           "output_gate", "output_gate_bwd", "prologue", "prologue_bwd"] + \
    list(binding.SIGNATURES)

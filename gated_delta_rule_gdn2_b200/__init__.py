"""B200 (sm_100a) Gated DeltaNet-2 sequence mixer.

The computation lives in ``libgdn2.so`` (hand-written CUDA kernels behind the
C ABI of include/gdn2.h); this package is its ctypes binding.  The library is
loaded on first use, and every call fails loudly if it has not been built
(``python -m gated_delta_rule_gdn2_b200.build``): there is no other code path.
"""
from .binding import (GDN2_BF16, GDN2_FP32, LIB_PATH, STATUS, Gdn2Error, chunk_bwd, chunk_fwd,
                      decode_step, gdn2_chunk_bwd, gdn2_chunk_bwd_workspace, gdn2_chunk_fwd,
                      gdn2_chunk_bwd_saved, gdn2_chunk_bwd_saved_workspace,
                      gdn2_chunk_fwd_noalloc, gdn2_chunk_fwd_save, gdn2_chunk_fwd_workspace,
                      gdn2_chunk_states_bytes, gdn2_decode_step, gdn2_get_device_status,
                      gdn2_status_string, gdn2_version, load)


__all__ = ["GDN2_BF16", "GDN2_FP32", "LIB_PATH", "STATUS", "Gdn2Error", "chunk_bwd", "chunk_fwd",
           "decode_step", "gdn2_chunk_bwd", "gdn2_chunk_bwd_workspace", "gdn2_chunk_fwd",
           "gdn2_chunk_bwd_saved", "gdn2_chunk_bwd_saved_workspace", "gdn2_chunk_fwd_noalloc",
           "gdn2_chunk_fwd_save", "gdn2_chunk_fwd_workspace", "gdn2_chunk_states_bytes", "gdn2_decode_step", "gdn2_get_device_status",
           "gdn2_status_string", "gdn2_version", "load"]

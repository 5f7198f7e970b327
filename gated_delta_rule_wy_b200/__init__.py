"""B200-native Gated Delta Rule-2 (GDR-2) token mixer.

The compute path is libgdr2.so (hand-written CUDA for sm_100a behind the C
ABI of ``include/gdr2.h``); ``binding`` exposes the same entry points on torch
tensors. ``inputs`` draws the seeded synthetic workloads. Importing the
package does not load the CUDA library; the first call does, and fails loudly
if it is missing.
"""
from .binding import (GDR2Error, gdr2_abi_version, gdr2_backward, gdr2_backward_noalloc,  # noqa: F401
                      gdr2_backward_workspace_bytes, gdr2_block_prologue, gdr2_decode_step, gdr2_forward,
                      gdr2_forward_varlen, gdr2_forward_varlen_workspace_bytes, gdr2_forward_workspace_bytes,
                      gdr2_gate_activations, gdr2_last_error, gdr2_segment_states, gdr2_short_conv_silu,
                      gdr2_sync_status, load_library)
from .segments import gdr2_forward_segmented, gdr2_forward_sequence_parallel  # noqa: F401

__all__ = ["GDR2Error", "gdr2_abi_version", "gdr2_backward", "gdr2_backward_noalloc",
           "gdr2_backward_workspace_bytes", "gdr2_forward_workspace_bytes",
           "gdr2_decode_step", "gdr2_forward", "gdr2_forward_varlen", "gdr2_forward_varlen_workspace_bytes",
           "gdr2_last_error", "gdr2_sync_status", "load_library", "gdr2_block_prologue", "gdr2_gate_activations",
           "gdr2_short_conv_silu", "gdr2_segment_states", "gdr2_forward_segmented", "gdr2_forward_sequence_parallel"]

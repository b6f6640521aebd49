"""Looped gated delta-rule (GDN) mixer for NVIDIA B200 (sm_100a).

The library is the C-ABI shared object ``libgdn.so`` (declared in
``include/gdn.h``), built from ``csrc/`` by ``looped_linear_attention_b200.build``.
This package is its thin Python binding plus the seeded workload generators:

    gdn_chunk_fwd    chunkwise prefill over packed / variable-length sequences
    gdn_decode_step  one token per state slot, in-place state update
    GDN_CHANNEL_GATE flag: the per-channel (diagonal) gate variant, KDA
    loop_residual    h = h_tilde + rho (.) h_prev
    swa_fwd          sliding-window causal softmax attention (the hybrid loops' window mixer)
    LoopedPrefill    T loops of projection -> GDN -> loop residual
    HostPipeline     looped-prefill steps on pinned host buffers, copies overlapped

No compute runs in Python: if the library is missing, every entry point raises.
"""
from ._binding import (GDN_BF16, GDN_ERR_CUDA, GDN_ERR_INVALID, GDN_ERR_TIMEOUT,
                       GDN_ERR_UNSUPPORTED, GDN_ERR_WORKSPACE, GDN_F32, GDN_OK, GDN_PRECISE,
                       GDN_QK_L2NORM, GDN_SINGLE_PASS, GDN_CHANNEL_GATE, GDN_TEST_WAIT_TIMEOUT, GdnError, gdn_chunk_bwd,
                       gdn_chunk_fwd, gdn_decode_step,
                       gdn_get_device_status, library, loop_residual, prefill_schedule, prefill_workspace_bytes,
                       status_string, swa_fwd, version)
from .looped import HostPipeline, LoopedPrefill, stack_weights

__all__ = [
    "gdn_chunk_fwd", "gdn_chunk_bwd", "gdn_decode_step", "loop_residual", "swa_fwd",
    "gdn_get_device_status",
    "prefill_schedule", "prefill_workspace_bytes",
    "LoopedPrefill", "HostPipeline", "stack_weights", "GdnError", "library", "status_string", "version",
    "GDN_OK", "GDN_ERR_INVALID", "GDN_ERR_UNSUPPORTED", "GDN_ERR_CUDA", "GDN_ERR_TIMEOUT",
    "GDN_ERR_WORKSPACE", "GDN_F32", "GDN_BF16", "GDN_QK_L2NORM", "GDN_PRECISE",
    "GDN_SINGLE_PASS", "GDN_CHANNEL_GATE", "GDN_TEST_WAIT_TIMEOUT",
]

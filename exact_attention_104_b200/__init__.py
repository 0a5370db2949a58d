"""Exact attention (FlashAttention-style forward and backward) for NVIDIA B200.

The compute lives in ``libfa_b200.so`` (hand-written sm_100a CUDA behind the C
ABI declared in ``include/fa.h``); this package only marshals arguments.
"""

from .binding import (  # noqa: F401
    FAError,
    fa_fwd,
    fa_fwd_pair,
    fa_bwd,
    fa_bwd_workspace_bytes,
    fa_device_status,
    fa_profile_next,
    fa_status_string,
    attention_forward,
    attention_backward,
    attention_decode,
    attention_forward_varlen,
    attention_backward_varlen,
    fa_fwd_varlen,
    fa_bwd_varlen,
    fa_fwd_varlen_workspace_bytes,
    fa_bwd_varlen_workspace_bytes,
    fa_fwd_decode,
    fa_decode_workspace_bytes,
    lib,
    LIB_PATH,
)

"""Exact RoPE / LeRoPE softmax attention (forward, loss, backward) for B200.

The compute lives in ``librope_attn.so`` (hand-written sm_100a CUDA behind the
C ABI in ``include/rope_attn.h``); :mod:`.binding` is its ctypes binding.
"""
from .binding import (  # noqa: F401
    problem, rope_attn_alpha_adam, rope_attn_bwd, rope_attn_bwd_saved,
    rope_attn_device_status, rope_attn_fwd, rope_attn_fwd_noalloc, rope_attn_loss,
    rope_attn_proj_bwd, rope_attn_proj_fwd, rope_attn_proj_workspace_bytes,
    rope_attn_spectrum, rope_attn_spectrum_workspace_bytes, rope_attn_timing_enable,
    rope_attn_timing_read, rope_attn_workspace_bytes, workspace)

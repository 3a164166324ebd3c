"""B200 (sm_100a) fused causal GQA attention, forward and backward.

The compute lives in ``libaxis_attn.so`` (hand-written CUDA, C ABI in
``include/axis_attn.h``); ``binding`` is its ctypes front end.  Importing the
package does not load the library; the first call does, and raises if it is
missing (there is no CPU fallback).
"""
from .binding import (  # noqa: F401
    EXPORTS,
    AxisAttnError,
    attention_backward,
    attention_backward_rope,
    attention_decode,
    attention_forward,
    attention_forward_rope,
    axis_attn_bwd,
    axis_attn_bwd_det,
    axis_attn_bwd_det_workspace_bytes,
    axis_attn_bwd_finalize,
    axis_attn_bwd_main,
    axis_attn_bwd_noalloc,
    axis_attn_bwd_prepare,
    axis_attn_bwd_rope,
    axis_attn_bwd_workspace_bytes,
    axis_attn_bwd_head_split,
    axis_attn_decode,
    axis_attn_decode_hnd,
    axis_attn_decode_q,
    axis_attn_decode_q_workspace_bytes,
    axis_attn_decode_workspace_bytes,
    axis_attn_fwd,
    axis_attn_fwd_rope,
    axis_attn_get_status,
    axis_attn_last_status_word,
    axis_attn_rope,
    axis_attn_rope_table,
    axis_attn_strerror,
    check_status,
    library_path,
    load,
    rope_table,
)

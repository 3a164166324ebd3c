"""fp64 CPU oracle for causal GQA attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never does.
"""
from .oracle import (  # noqa: F401
    attn_bwd,
    attn_decode,
    attn_decode_q,
    attn_bwd_dkdv_rows,
    attn_bwd_dq_rows,
    attn_fwd,
    attn_fwd_rows,
    build,
    max_threads,
    probs_row,
    rope,
)

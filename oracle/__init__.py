"""fp64 CPU oracle for exact attention.  Test infrastructure only (see attention.py)."""
from .attention import (  # noqa: F401
    chunk_positions,
    scores,
    softmax_rows,
    attention_head,
    attention_head_tiled,
    attention_bwd_head,
    attention_bwd_dq_rows,
    attention_fwd,
    attention_bwd,
)

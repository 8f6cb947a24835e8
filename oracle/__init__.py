"""fp64 CPU oracle for exact attention (test infrastructure only; see attention.py)."""

from .attention import (  # noqa: F401
    attention_bwd,
    attention_bwd_head,
    attention_fwd,
    attention_fwd_head,
    attention_fwd_partial,
    attention_fwd_rows,
    attention_fwd_head_tiled,
    lse_merge,
    softmax_rows,
)
from .dropout import (  # noqa: F401
    attention_bwd_dropout,
    attention_fwd_dropout,
    drop_threshold,
    keep_mask,
    keep_scale,
    philox4x32_10,
)

"""fp64 CPU oracle for exact softmax attention (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import this package. It is independent of the CUDA library.
"""
from .attention import (  # noqa: F401
    attn_bwd_block_ref,
    attn_bwd_ref,
    attn_dkdv_cols_ref,
    attn_dq_rows_ref,
    attn_fwd_block_ref,
    attn_fwd_ref,
    attn_fwd_rows_ref,
    attn_probs_ref,
    attn_scores_ref,
)
from .dropout import (  # noqa: F401
    attn_dropout_bwd_ref,
    attn_dropout_fwd_ref,
    dropout_keep_mask,
    keep_threshold,
    philox4x32_10,
)

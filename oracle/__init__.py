"""fp64 CPU oracle for exact attention (test infrastructure; see attention.py)."""
from .attention import (  # noqa: F401
    as_f64,
    attention_bwd,
    attention_bwd_sampled,
    attention_bwd_gqa,
    attention_fwd,
    attention_fwd_gqa,
    attention_fwd_blockwise,
    attention_fwd_decode,
    attention_fwd_general,
    attention_bwd_general,
    attention_fwd_varlen,
    attention_bwd_varlen,
    attention_fwd_rows,
    bwd_operand_rounding_bound,
    softmax_merge,
)

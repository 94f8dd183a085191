"""fp64 CPU oracle (test infrastructure only; never imported by the product path)."""
from .attention_ref import (  # noqa: F401
    attention_bwd,
    attention_bwd_gqa,
    attention_bwd_rows_dq,
    attention_decode,
    attention_fwd,
    attention_fwd_heads,
    attention_fwd_online,
    attention_fwd_rows,
    softmax_probs,
)
from .brute import brute_bwd, brute_decode, brute_fwd  # noqa: F401

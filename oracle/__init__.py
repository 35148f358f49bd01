"""fp64 CPU oracle (test infrastructure only; see ``oracle.attention``)."""
from .attention import (  # noqa: F401
    allowed_mask, scaled_scores, attention_probs, attention_forward,
    attention_forward_online, delta_rowsum, attention_backward,
    attention_forward_rows, attention_backward_dq_rows, attention_head,
)

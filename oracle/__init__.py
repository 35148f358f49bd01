"""fp64 CPU oracle (test infrastructure only; see ``oracle.attention``, and
``oracle.fp8`` for the e4m3 forward)."""
from .attention import (  # noqa: F401
    allowed_mask, scaled_scores, attention_probs, attention_forward,
    attention_forward_online, delta_rowsum, attention_backward,
    attention_forward_rows, attention_backward_dq_rows, attention_head,
)

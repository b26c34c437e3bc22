"""CPU oracle for exact attention (test infrastructure only; see attention_ref)."""
from .attention_ref import (  # noqa: F401
    attention_forward, attention_forward_head, attention_backward, attention_backward_head,
    scaled_scores, softmax_rows, allowed_mask, two_block_softmax, online_softmax_elementwise,
    online_softmax_blocks, standard_attention_counted, brute_force_attention, e4m3_decode,
    attention_forward_fp8,
)

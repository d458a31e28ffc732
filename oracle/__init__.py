"""Float64 CPU oracle for exact attention (test infrastructure only).

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package; the CUDA library never does.
"""
from .attention_ref import (  # noqa: F401
    attention_backward,
    attention_backward_dq_rows,
    attention_backward_varlen,
    attention_bruteforce,
    attention_forward,
    attention_forward_varlen,
    attention_forward_rows,
    attention_head,
    attention_head_bwd,
    capped,
    causal_visible,
    dense_score_matrix_bytes,
    dense_score_matrix_cells,
    online_softmax_attention_head,
    scores,
    softmax_rows,
    to_f64,
    visible,
)

"""CPU float64 oracle for scaled-dot-product attention (test infrastructure).

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA path never does.
"""
from .sdpa_oracle import (  # noqa: F401
    alibi_slope_gradient,
    attention_backward,
    attention_backward_packed,
    attention_forward,
    attention_forward_packed,
    attention_probs,
    dense_bias_gradient,
    fire_gradients,
    fire_table,
    head_scores,
    packed_positions,
    packed_visibility_mask,
    rel_table_gradient,
    t5_relative_bucket,
    t5_table_gradient,
    visibility_mask,
)

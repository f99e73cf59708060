"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
``--impl reference`` legs may import this package.  The CUDA library and its
Python binding never import it; the two share no code.  See
``attention_fp64.py`` for the definition it follows and its citations.
"""
from .attention_fp64 import (  # noqa: F401
    brute_fwd,
    brute_fwd_general,
    dropout_multiplier,
    dropout_threshold,
    finite_diff_grads_general,
    kv_head_of,
    philox4x32_10,
    ref_bwd_general,
    ref_dq_general_rows,
    ref_fwd_general,
    ref_fwd_general_rows,
    softmax_rows_masked,
    causal_keep,
    finite_diff_grads,
    ref_bwd,
    ref_bwd_head,
    ref_dq_rows,
    ref_fwd,
    ref_fwd_rows,
    ref_probs,
    scores,
    softmax_grad,
    softmax_rows,
)

"""fp64 CPU oracle for exact attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline and
``--impl reference`` legs may import this package.  The CUDA library and its
Python binding never import it; the two share no code.  See
``attention_fp64.py`` for the definition it follows and its citations.
"""
from .attention_fp64 import (  # noqa: F401
    brute_fwd,
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

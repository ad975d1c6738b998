"""fp64 CPU oracle for exact softmax attention (test infrastructure only).

This package is test infrastructure.  Only the tests, ``__graft_entry__.smoke()``
and the bench's CPU-baseline / reference arm may import it; the product path
(the C-ABI library and its Python binding) never calls it and has no CPU
fallback.  It shares no code with the CUDA path.

Every output of every function here is pinned by the CPU tests in
``tests/test_oracle.py`` (worked closed forms, finite differences, invariants,
an independent autograd library, large-logit overflow behaviour); nothing is
"parity unpinned".
"""

from .attention import (  # noqa: F401
    scores,
    softmax_rows,
    attention_forward_2d,
    attention_backward_2d,
    attention_forward,
    attention_backward,
    attention_forward_gqa,
    attention_backward_gqa,
    attention_forward_rows,
    attention_backward_rows,
    attention_backward_keys,
    chunked_forward_2d,
    combine_partials,
    combine_two_blocks,
)

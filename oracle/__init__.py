"""Float64 CPU oracle for fused linear cross-entropy (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline / reference
legs import this package. The CUDA library and its Python binding never do.
"""
from .flce_oracle import (  # noqa: F401
    count_valid,
    cross_entropy,
    dlogits,
    flce,
    flce_brute_force,
    flce_grad_W_rows,
    flce_rows,
    logits,
    row_logsumexp,
    valid_mask,
)

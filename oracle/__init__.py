"""fp64 CPU oracle for exact attention (test infrastructure only; see oracle.py)."""
from .oracle import (  # noqa: F401
    SOURCE,
    Oracle,
    backward,
    backward_dkdv_rows,
    backward_dq_rows,
    build,
    default,
    forward,
    forward_rows,
    num_threads,
    probs,
    set_num_threads,
)

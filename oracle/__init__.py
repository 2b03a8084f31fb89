"""Float64 CPU oracle for dilated attention.

TEST INFRASTRUCTURE ONLY. Nothing in the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may use it. It shares no code with the CUDA path.
"""
from .dilated import (  # noqa: F401
    kept_rows,
    selection_signature,
    fwd,
    fwd_head,
    fwd_per_pattern,
    bwd,
    bwd_head,
    fwd_rows,
    bwd_rows,
    multiplicity,
    fwd_bruteforce,
    effective_pairs,
)

"""fp64 CPU oracle for the StreamKL attention KL divergence.

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU-baseline leg
may import this package; the product path (the CUDA library and its binding) never does,
and the two share no code.

Two independent restatements of the method live here:

* ``streamkl_oracle.c`` (loaded through ctypes): the per-row two-pass definition of the
  attention KL and its gradients in double precision, plus a literal run of the pages'
  five-scalar online recurrence (``fwd_streaming``).
* ``brute``: materialises P1 and P2 as full matrices with numpy (small inputs only).

See the header of ``streamkl_oracle.c`` for the formulas and the passages they follow.
"""
from .oracle import (  # noqa: F401
    build,
    fwd,
    fwd_rows,
    fwd_streaming,
    bwd,
    bwd_dq_rows,
    bwd_dk_keys,
    bwd_dk_keys_stats,
    num_threads,
    set_num_threads,
)
from . import brute  # noqa: F401

"""CPU oracle for the Flint MoE-layer forward (fp64, numpy).

Test infrastructure: only the test suite, the package smoke check and the
benchmark's CPU-baseline leg may import it. The CUDA library and its Python
binding never do.

Parity status: every function in flint_moe_ref is pinned by a `-m "not gpu"`
test against something other than itself (closed forms, invariants, library
routines for the special cases, brute force on tiny inputs); see
tests/test_oracle_pins.py. The whole layer on Flint's trained weights is
parity unpinned: neither those weights nor the pages' own FP64 forward are
available, and none is needed for the synthetic workloads.
"""
from . import flint_moe_ref  # noqa: F401

"""CPU oracle for the MoE expert-MLP hot path — TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. The product path (the CUDA library and its
Python binding) never calls it, and this package imports nothing from the product.

Everything is plain numpy in float64 (plus exact table-driven MXFP8 encoding), written
to be checked by eye against the pages it follows:

* "Efficient MoE training for biological foundation models" (NVIDIA developer blog, as
  summarised on sitech.ge) — section "Grouped experts instead of a Python loop": experts
  process the tokens routed to them, grouped with per-expert counts (``split_sizes``);
  the routing weights are applied inside the fused GroupedMLP kernel.
* The same post on news.bpdata.com — section 1) "fragmented expert kernels" (grouped
  GEMM over per-expert token counts, equivalent to the per-expert loop), section 2)
  (MXFP8: one scale per block of 32 consecutive values) and section 3) (the fused chain
  GroupedLinear -> ScaledSwiGLU -> GroupedLinear, 16-bit master weights).

Where the pages leave a step open the oracle takes the plainest reading; the readings
are listed in the module docstrings of :mod:`oracle.moe` and :mod:`oracle.mxfp8`.

Parity status: every function here is pinned by ``tests/test_oracle_*.py`` against
closed forms, library routines (torch fp64 autograd, ml_dtypes casts), brute force or
hand-derived fixtures in ``tests/golden/``.
"""
from . import mxfp8, moe  # noqa: F401

__all__ = ["mxfp8", "moe"]

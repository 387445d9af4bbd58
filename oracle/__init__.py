"""Float64 CPU oracle for the OFT-adapted linear over a frozen low-precision base.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check in the graft entry
module and the CPU-baseline leg of the benchmark may import this package.  The
product path (the CUDA library and its Python binding) never calls into it and
shares no code with it: no kernels, headers, helpers, tables or constant
generators.

Modules:
  codecs   -- bf16 rounding, INT4 / FP8 e4m3 / MXFP4 (e2m1 + e8m0) decoding and
              group-wise dequantisation.
  oft_ref  -- Cayley rotation build, split-projection forward, and the adapter
              backward (dX and dQ through the Cayley map).
  moe_ref  -- top-k routing with softmax gating, bucketing, active-expert
              chunking, and the chunked MoE forward.

Every function is a plain restatement of the definition it cites; numpy's
matmul and linear solve are the only library steps.  Each is pinned by the
CPU tests (tests/test_oracle_*.py) to facts that do not come from the oracle
itself: closed forms, library codecs, finite differences, invariants, brute
force.  Parity pins are listed in the module docstrings.
"""

from . import codecs, oft_ref, moe_ref  # noqa: F401

"""Seeded synthetic inputs for the OFT linear and the chunked-MoE OFT layer.

This package is shared by the float64 oracle tests, the GPU parity tests and
the benchmark.  It only draws inputs (activations, packed low-precision weight
codes and their scales, adapter parameters, upstream gradients, router
logits); it holds none of the method's arithmetic (no dequantisation, no
rotation, no GEMM, no routing).
"""

from .workloads import (  # noqa: F401
    LinearSpec,
    MoESpec,
    LINEAR_CONFIGS,
    MOE_CONFIGS,
    make_linear_case,
    make_moe_case,
    make_moe_down,
    make_moe_grad,
    make_moe_router,
    split_offsets,
)

"""B200-native (sm_100a) OFT hot path: an orthogonal adapter in front of a frozen
INT4 / FP8 / MXFP4 linear layer, its backward, and the active-expert-chunked MoE
variant.  The compute lives in liboft.so (C ABI: include/oft.h); this package is
the Python binding over it."""

from .binding import (  # noqa: F401
    OFTError,
    Weight,
    library_path,
    moe_chunked_oft_bwd,
    moe_chunked_oft_bwd_workspace,
    moe_chunked_oft_fwd,
    moe_chunked_oft_layer_fwd,
    moe_chunked_oft_layer_workspace,
    moe_chunked_oft_workspace,
    moe_fused_oft_fwd,
    moe_fused_oft_workspace,
    oft_build_rotation,
    oft_cayley_backward,
    oft_check_device,
    oft_debug_bounded_wait,
    oft_dequant_weight,
    oft_linear_bwd,
    oft_linear_bwd_workspace,
    oft_linear_fwd,
    oft_linear_fwd_noalloc,
    oft_linear_fwd_weight_side,
    oft_linear_fwd_weight_side_workspace,
    oft_linear_fwd_workspace,
    oft_moe_chunk_dequant,
    oft_rotate,
    oft_set_gemm_mode,
    profile,
    version,
)
from .slots import AdapterSlots  # noqa: F401,E402

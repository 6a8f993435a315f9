"""Activation-sparse gated-epilogue FFN for NVIDIA B200 (sm_100a).

Thin Python binding over the C-ABI library ``libsge.so`` (declared in
``include/sge.h``).  Every step of the computation runs in the library's CUDA
kernels; this package only marshals torch tensors (device memory, streams)
into pointers and sizes.  There is no CPU fallback: if the library is missing
or a tensor is not on a CUDA device, the call raises.
"""
from .binding import (  # noqa: F401
    SGE_BF16, SGE_F32, TwELL, LibraryError, library, library_path,
    twell_gate_pack, twell_fused_up_down, twell_ffn_forward, dense_ffn_fwd, new_diag,
    fused_workspace, Hybrid, hybrid_pack, hybrid_ffn_fwd, hybrid_fwd_workspace,
    hybrid_ffn_bwd, hybrid_bwd_workspace, interleave_up_down, twell_hybrid_up_down, routed_workspace,
    transpose_up_gate, debug_flags,
)

__all__ = [
    "SGE_BF16", "SGE_F32", "TwELL", "LibraryError", "library", "library_path",
    "twell_gate_pack", "twell_fused_up_down", "twell_ffn_forward", "dense_ffn_fwd", "new_diag",
    "fused_workspace", "Hybrid", "hybrid_pack", "hybrid_ffn_fwd", "hybrid_fwd_workspace",
    "hybrid_ffn_bwd", "hybrid_bwd_workspace", "interleave_up_down", "twell_hybrid_up_down",
    "routed_workspace", "transpose_up_gate", "debug_flags",
]

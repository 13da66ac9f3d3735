"""B200-native block-sparse attention with top-k summary routing.

The computation runs in ``lib/libssa.so`` (hand-written sm_100a CUDA kernels
behind the C ABI of ``include/ssa.h``); this package is its ctypes binding.
There is no CPU fallback: every call needs the built library and a CUDA device.
"""
from .abi import (  # noqa: F401
    SSAError,
    decode_width,
    ssa_debug_wait_timeout,
    load_library,
    prefill,
    route_width,
    ssa_block_summary,
    ssa_check_device_error,
    ssa_decode,
    ssa_decode_append,
    ssa_decode_noalloc,
    ssa_decode_paged,
    ssa_decode_append_paged,
    ssa_decode_workspace_size,
    ssa_device_error,
    entmax_width,
    ssa_learned_summary,
    ssa_route_entmax,
    ssa_route_hierarchical,
    ssa_decode_per_head,
    ssa_decode_per_head_workspace_size,
    ssa_sparse_attn_fwd_prior,
    ssa_route,
    ssa_sparse_attn_bwd,
    ssa_sparse_attn_bwd_workspace_size,
    ssa_sparse_attn_fwd,
    ssa_sparse_attn_uses_tensor_cores,
)

__version__ = "0.1.0"

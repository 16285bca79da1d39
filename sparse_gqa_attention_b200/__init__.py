"""Elastic Attention prefill path on B200 (sm_100a).

The compute lives in libea.so (CUDA kernels behind the C ABI in include/ea.h);
``abi`` is its Python binding.  PyTorch is used for device memory and streams.
"""
from .abi import (  # noqa: F401
    EAError, Pattern,
    ea_router, ea_router_workspace_size, ea_router_static_scratch,
    ea_hybrid_attn_prefill, ea_hybrid_attn_prefill_chunk, ea_build_schedule, ea_attn_scheduled, ea_attn_workspace_size,
    ea_effective_sparsity, ea_workspace_status, ea_status_string,
    EA_FULL, EA_STREAMING, EA_BLOCK_SPARSE,
)

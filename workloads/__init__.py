"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This package holds the input generators only: random draws, bf16 rounding of
those draws, the block-sparse layout draw and the workload shapes.  It holds
none of the method's arithmetic (no pooling, no router MLP, no attention, no
sparsity counting); the CUDA path and the CPU oracle each compute those on
their own.
"""
from .generate import (  # noqa: F401
    FULL, STREAMING, BLOCK_SPARSE, STREAMING_BLOCKS,
    WORKLOADS, Workload, Pattern,
    bf16_bits_from_f32, f32_from_bf16_bits,
    attention_inputs, hidden_states, router_weights, block_layout, pattern_for,
    forced_head_mode, routing_targets, load_router_tuning, positional_component, probe_layer_inputs,
)

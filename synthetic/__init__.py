"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the CPU oracle.

This package draws random numbers and lays them out; it holds none of the
arithmetic of the gated block-sparse decode itself (no pooling, projection,
RoPE, scoring, selection or attention).
"""

from .inputs import (  # noqa: F401
    CONFIGS,
    SWEEP_SPARSITIES,
    DecodeConfig,
    DecodeInputs,
    bf16_bits_from_f32,
    bf16_bits_to_f32,
    config,
    make_block_lists,
    make_inputs,
    make_logits,
    make_pair_inputs,
    make_step_query,
    paged_view,
    scale_gate_weights,
    sweep_budget,
)

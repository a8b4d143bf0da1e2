"""Seeded synthetic inputs for the compressed-expert MoE layer.

This package draws random bytes, codes and floats in the shapes of the
workloads; it performs none of the layer's arithmetic (no decode, no
matmul, no activation).  Both the oracle tests and the CUDA path take
their inputs from here, so neither side ever manufactures the other's
inputs.
"""
from .gen import (  # noqa: F401
    CONFIGS,
    LayerCfg,
    Layer,
    get_cfg,
    gen_layer,
    gen_routing,
    gen_activations,
    gen_router,
    gen_disjoint_routing_schedule,
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    idx13_row_bytes,
    gvq1_code_row_bytes,
    e4m3_bytes_from_f32,
)

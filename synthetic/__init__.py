"""Seeded synthetic inputs for the routed low-bit MoE layer.

This package only draws random tensors and encodes them into the stored
weight formats (MLX-style affine packs, mxfp4 packs, the tid2eid table).  It
holds none of the layer's arithmetic: no routing, no dequantisation, no
contraction.  Both the CPU oracle's tests and the CUDA path's tests/bench
consume what it produces.
"""
from .moe_inputs import (  # noqa: F401
    CONFIGS,
    FP8_CONFIGS,
    Fp8Inputs,
    make_fp8_inputs,
    HC_CONFIGS,
    HcInputs,
    make_hc_inputs,
    QMat,
    MoEInputs,
    make_inputs,
    make_custom,
    pack_bits,
    quantize_affine,
)

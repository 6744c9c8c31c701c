"""Seeded synthetic workloads for the TwELL gated-FFN hot path.

This package only draws random numbers and rounds them to bfloat16 storage.
It holds none of the FFN or packing arithmetic, so both the CUDA path and the
CPU oracle can consume its output without sharing any of the method's code.
"""

from .workloads import (  # noqa: F401
    WORKLOADS,
    Workload,
    bf16_bits_from_f64,
    bf16_bits_to_f32,
    gate_bias_for_activity,
    make_inputs,
    sweep_k,
    sweep_workload,
)

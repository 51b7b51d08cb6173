"""Seeded synthetic input generation (no arithmetic of the method lives here)."""
from .inputs import (  # noqa: F401
    WORKLOADS,
    Workload,
    bf16_bits_to_f32,
    bf16_bits_to_f64,
    f32_to_bf16_bits,
    make_cotangent,
    make_inputs,
    make_workload_inputs,
)

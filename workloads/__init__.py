"""Seeded synthetic workloads shared by the tests, the benchmark and the oracle (random draws only)."""
from .synthetic import (Workload, WORKLOADS, INT4_SWEEP_TOKENS, workload, make_inputs, Inputs,
                        bf16_bits_from_f64, bf16_bits_to_f32)

__all__ = ["Workload", "WORKLOADS", "INT4_SWEEP_TOKENS", "workload", "make_inputs", "Inputs",
           "bf16_bits_from_f64", "bf16_bits_to_f32"]

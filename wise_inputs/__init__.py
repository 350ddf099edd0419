"""Seeded synthetic workloads shared by the oracle, the tests and the benchmark."""
from .generator import (BLOCK, CONFIGS, SUPPLEMENTARY, WorkloadConfig, HeadStream, all_heads, iter_steps,
                        generate_all_steps, f32_to_bf16_bits, bf16_bits_to_f32,
                        bf16_bits_to_f64)

__all__ = ["BLOCK", "CONFIGS", "SUPPLEMENTARY", "WorkloadConfig", "HeadStream", "all_heads", "iter_steps",
           "generate_all_steps", "f32_to_bf16_bits", "bf16_bits_to_f32", "bf16_bits_to_f64"]

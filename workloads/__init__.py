"""Seeded synthetic SANA-WM-shaped GDN workloads (sizes and input generation only)."""

from .configs import CONFIGS, TINY, BLOCK, CLIP241, MINUTE, SESSIONS, Workload, long_memory
from .synth import (Fp8Inputs, Inputs, bf16_bits, bf16_round, draw, e4m3_encode, make_fp8_inputs,
                    make_inputs, make_session_blocks, to_fp8, v_scale_for)

__all__ = ["CONFIGS", "TINY", "BLOCK", "CLIP241", "MINUTE", "SESSIONS", "Workload",
           "long_memory", "Inputs", "bf16_bits", "bf16_round", "draw", "make_inputs",
           "make_session_blocks", "Fp8Inputs", "e4m3_encode", "make_fp8_inputs", "to_fp8",
           "v_scale_for"]

"""Seeded synthetic SANA-WM-shaped GDN workloads (sizes and input generation only)."""

from .configs import CONFIGS, TINY, BLOCK, CLIP241, MINUTE, SESSIONS, Workload, long_memory
from .synth import Inputs, bf16_bits, bf16_round, draw, make_inputs, make_session_blocks

__all__ = ["CONFIGS", "TINY", "BLOCK", "CLIP241", "MINUTE", "SESSIONS", "Workload",
           "long_memory", "Inputs", "bf16_bits", "bf16_round", "draw", "make_inputs",
           "make_session_blocks"]

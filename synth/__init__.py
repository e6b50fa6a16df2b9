"""Seeded synthetic inputs shared by the CPU oracle and the CUDA path.

This module only draws random numbers and shapes them like the workloads the
pages describe (per-token activations with a few outlier channels, N(0, 0.02)
weights with rare large entries, router logits with a Zipf skew).  It holds
none of the quantization / GEMM / routing arithmetic: both sides receive the
exact same bytes from here and compute independently.

Draw order inside one generator (fixed, so a seed names one input set):
  X, outlier-channel choice, W (per matrix), weight-outlier mask, logits,
  Zipf rank permutation.
"""
from .inputs import (  # noqa: F401
    LinearInputs,
    MoEInputs,
    gen_linear,
    gen_moe_activations,
    gen_expert_weight,
    zipf_logits,
    CONFIGS,
)

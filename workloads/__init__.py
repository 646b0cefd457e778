"""Seeded synthetic inputs for the fused chunked top-K KL loss.

This package only draws random inputs (student hidden states H, LM-head
weight W, an offline teacher top-K cache and a loss mask) with the shapes
and value distributions of the workloads that "Efficient Knowledge
Distillation for LLMs: Offline Top-K Logits and a Fused Chunked KL Loss"
measures on.  It computes nothing of the loss itself.  Both the fp64 oracle
(tests only) and the CUDA path consume what it returns.
"""

from .configs import CONFIGS, Config, get_config
from .gen import make_inputs, sample_distinct

__all__ = ["CONFIGS", "Config", "get_config", "make_inputs", "sample_distinct"]

"""Seeded synthetic workloads for the grouped NF4 W4A16 expert GEMM.

This module only draws random numbers and shapes them into the inputs the
method consumes. It holds none of the method's arithmetic (no NF4 table, no
decode, no contraction), so both the CUDA path and the CPU oracle can take
their inputs from here without sharing any code with each other.

Workloads follow the MoE shapes of the grouped-nf4-gemm README (the
"The claim" section lists the census models: OLMoE, Qwen3-30B, GPT-OSS-120B,
and the k=2 large shapes such as Mixtral-8x22B). No dataset or checkpoint is
involved: weights are N(0, 0.02) fp32 draws (quantised to NF4 by the caller),
activations are N(0, 1) rounded to bf16, and routing is drawn per workload.
"""
from .workloads import (  # noqa: F401
    WORKLOADS,
    Workload,
    Gemm,
    seed_streams,
    routing,
    activations_bf16,
    expert_weights_f32,
    random_packed_stack,
    bf16_bits_to_f32,
)

"""Seeded synthetic inputs for the sparse-prefill path.

This package holds the workload definitions (shapes, budgets, DCA constants,
refinement threshold) and the seeded generator of pre-RoPE Q, K, V tensors. It
contains none of the method's arithmetic (no RoPE, softmax, selection or
attention): both the CPU oracle's tests and the CUDA path consume the same
tensors it produces.
"""
from .configs import WORKLOADS, Workload, small_workload
from .gen import generate_head, generate_layer, planted_positions, structure

__all__ = [
    "WORKLOADS",
    "Workload",
    "small_workload",
    "generate_head",
    "generate_layer",
    "planted_positions",
    "structure",
]

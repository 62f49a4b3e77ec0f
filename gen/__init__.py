"""Seeded synthetic workloads for block-sparse video attention.

This package is the one piece of code that both the CUDA path's tests/bench
and the CPU oracle use: it describes the workload shapes and draws seeded
Q/K/V tensors with the structure of video-DiT activations, and seeded
stand-ins for trained gate matrices. It contains no step of the attention
method itself (no layout, pooling, selection or softmax).
"""
from .configs import CONFIGS, SWEEP_KEEP_RATIOS, config, derived_sizes
from .synth import make_gate, make_qkv, make_tensor, layer_keep_schedule

__all__ = ["CONFIGS", "SWEEP_KEEP_RATIOS", "config", "derived_sizes",
           "make_gate", "make_qkv", "make_tensor", "layer_keep_schedule"]

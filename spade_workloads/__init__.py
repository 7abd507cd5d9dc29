"""Seeded synthetic workloads shaped like the video-DiT attention layers SPADE
is evaluated on (Wan 2.1 / Hunyuan-Video at 720p).

This package holds shapes and random-number generation only: none of the
method's arithmetic lives here.  Both the CPU oracle and the CUDA path draw
their inputs from it, so both see bit-identical tensors.
"""
from .configs import CONFIGS, Workload, Scheme, flat_scheme, get_config, config_names
from .gen import make_qkv, splitmix64, counter_uniform, counter_normal

__all__ = [
    "CONFIGS", "Workload", "Scheme", "flat_scheme", "get_config", "config_names",
    "make_qkv", "splitmix64", "counter_uniform", "counter_normal",
]

"""Seeded synthetic workloads for the hybrid compressed-attention hot path.

This package only draws random tensors and describes workload shapes.  It
holds none of the method's arithmetic: both the CUDA path and the CPU oracle
consume what it produces.
"""
from .configs import CONFIGS, WorkloadConfig, get_config  # noqa: F401
from .gen import (  # noqa: F401
    make_compress_inputs,
    make_indexer_inputs,
    make_attn_inputs,
    make_scores,
    make_topk_idx,
)

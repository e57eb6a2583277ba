"""Seeded synthetic workloads for the two-level sparse decode step.

This package only draws inputs: K/V caches, queries, label-channel indices and
query trajectories.  It holds none of the method's arithmetic (no scoring, no
selection, no quantisation, no attention), so that the CPU oracle and the CUDA
path can both consume the same bytes without sharing any computation.
"""

from .configs import CONFIGS, WorkloadConfig, get_config
from .gen import (
    bf16_bits_from_f32,
    f32_from_bf16_bits,
    RowInputs,
    gen_row,
    gen_queries,
    gen_query_trajectory,
    gen_label_channels,
    gen_outlier_channels,
    gen_kv,
)

__all__ = [
    "CONFIGS",
    "WorkloadConfig",
    "get_config",
    "bf16_bits_from_f32",
    "f32_from_bf16_bits",
    "RowInputs",
    "gen_row",
    "gen_queries",
    "gen_query_trajectory",
    "gen_label_channels",
    "gen_outlier_channels",
    "gen_kv",
]

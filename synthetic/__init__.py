"""Seeded synthetic video-token workloads shared by the oracle, the tests and the bench.

This package only draws inputs (Q, K, V and the workload's shape/parameter table).
It holds none of the attention method's arithmetic.
"""
from .video_tokens import CONFIGS, WorkloadConfig, make_inputs, token_grid_features

__all__ = ["CONFIGS", "WorkloadConfig", "make_inputs", "token_grid_features"]

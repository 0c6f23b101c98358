"""Seeded synthetic workloads for the block-sparse 3D-tile attention path.

This package is shared by the CUDA path's tests and benchmark and by the
CPU oracle. It draws random inputs and names the workload shapes; it holds
none of the method's arithmetic (no tiling, pooling, scoring, selection,
window test or attention).
"""
from .configs import CONFIGS, WorkloadConfig, tile_counts  # noqa: F401
from .gen import (  # noqa: F401
    make_qkv,
    perturb_step,
    window_params,
    window_scale,
    fixed_windows_tiny,
)

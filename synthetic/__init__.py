"""Seeded synthetic inputs for the TempCache step.

This package holds only input generation (random draws and rounding of the
draws to the storage precision). It contains none of the method's arithmetic,
so both the CPU oracle's tests and the CUDA path's tests may use it.
"""
from .workload import (  # noqa: F401
    CONFIGS,
    WorkloadConfig,
    Workload,
    round_to_bf16,
    draw_hyperplanes,
)
from .cross import (  # noqa: F401
    CROSS_CONFIGS,
    CrossConfig,
    CrossWorkload,
    draw_cross_hyperplanes,
)

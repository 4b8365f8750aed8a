"""Seeded synthetic KV-cache workloads shaped like the pages' models.

This package only draws inputs (keys, values, calibration vectors, queries);
it holds none of the compression arithmetic. Both the CUDA path and the CPU
oracle consume what it draws.
"""

from .workloads import CONFIGS, Workload, make_workload  # noqa: F401

"""Seeded synthetic inputs for the CSA / HCA attention layer.

This package is shared by the CUDA path's tests and benchmark and by the CPU
oracle. It holds shapes and random draws only: nothing in it computes any step
of the method (compression, indexing, selection or attention).
"""

from .workloads import WORKLOADS, Workload, make_inputs, decode_positions  # noqa: F401

"""Seeded synthetic inputs shared by the oracle tests, the GPU tests and the benchmark.

``gen`` is the counter-based random stream (NumPy), ``workloads`` the five decode
workloads and their planted structure, ``gpu`` the bulk GPU fill of the same stream.
"""
from . import gen, workloads  # noqa: F401

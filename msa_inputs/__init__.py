"""Seeded synthetic inputs (generator + workload definitions).

Serves both the fp64 oracle tests and the CUDA path's tests and benchmark;
holds none of the attention method's arithmetic.
"""
from . import rng, workloads  # noqa: F401

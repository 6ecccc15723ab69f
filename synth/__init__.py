"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This package only draws random numbers: Gaussian-mixture points and a random
initial centroid set.  It holds none of the clustering arithmetic (no
distances, no argmin, no means), so both the CUDA path and the CPU oracle can
consume the same tensors without sharing any of the method.
"""

from .mixtures import (  # noqa: F401
    WORKLOADS,
    Workload,
    make_points,
    make_problem,
    init_rows,
    pool_workload,
    instance_seed,
)

"""Seeded synthetic workloads shared by the CUDA path's tests/bench and the oracle.

This module only draws input data (Gaussian mixtures and their relatives). It
holds none of the e-means arithmetic: no assignment, no statistics, no update,
no rounding to the search format. Both sides receive the same bytes from here.
"""

from .synth import (  # noqa: F401
    WORKLOADS,
    Workload,
    blobs3,
    hand_shape,
    make,
    mixture_normalized,
    sift_like,
    subspace_mixture,
    isotropic_mixture,
)

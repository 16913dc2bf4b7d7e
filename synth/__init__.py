"""Seeded synthetic workloads shared by the oracle, the tests and the benchmark.

This package draws random numbers and nothing else: a weight matrix given by its
singular factors W = left . diag(sigma) . right^T, an activation matrix X and,
for the ALS start, a Gaussian matrix R0.
It contains none of the DyRA arithmetic (no truncation, no residual, no
projector, no solve); every consumer derives those on its own side.
"""

from .workloads import (  # noqa: F401
    CONFIGS,
    LLAMA_SWEEP,
    LayerSpec,
    Workload,
    gaussian_r0,
    generate,
    haar_orthonormal,
    make_activations,
    spec,
)

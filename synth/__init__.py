"""Seeded synthetic inputs shared by the oracle-side tests and the CUDA path.

This package holds random-number recipes only: no step of the quantisation
method lives here, so the CPU oracle and the GPU library can both consume the
same bytes without sharing any arithmetic of the method.
"""

from .gptq_inputs import (  # noqa: F401
    WORKLOADS,
    Workload,
    make_activations,
    make_weights,
    make_problem,
    workload,
    workload_inputs,
)

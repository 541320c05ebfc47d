"""Seeded synthetic inputs for the MLA latent-KV decode path.

This package only draws random numbers and lays them out (weights, hidden
states, cached latent rows, ragged lengths, paged block tables).  It holds
none of the method's arithmetic: no projection, no RoPE, no softmax.  Both
the fp64 oracle and the CUDA path consume what it produces, and neither
imports the other.
"""

from .workloads import (  # noqa: F401
    MLAShape,
    Workload,
    WorkloadData,
    SHAPES,
    WORKLOADS,
    generate,
    reduced,
    build_pool,
    build_row_scale,
    device_inputs,
)

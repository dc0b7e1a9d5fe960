"""Seeded synthetic workloads for the 1-bit Adam compressed-phase step.

This package holds only workload *shapes* (the chunk tables of the parameter
sets) and the seeded generators of the inputs (gradients, parameters, moment
state).  It contains none of the method's arithmetic, so both the CPU oracle
(test infrastructure) and the CUDA path draw their inputs from here.
"""

from .configs import WORKLOADS, Workload, get_workload  # noqa: F401
from .gen import (  # noqa: F401
    chunk_grads,
    chunk_state,
    chunk_groups,
    fill_grads,
    fill_grads_row,
    fill_state,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
    layer_multiplier,
    aux_normal,
    aux_bits,
    aux_uniform,
    BLOCK,
)

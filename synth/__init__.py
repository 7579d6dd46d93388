"""Seeded synthetic inputs for the SketchSSM decode path.

This package holds no arithmetic of the method itself: only shapes, rank tables,
bases and per-step random inputs.  Both the CPU oracle (tests) and the CUDA path
(tests, bench) draw their inputs from here, so the two sides always see the same
fp32 arrays.
"""
from .gen import (  # noqa: F401
    CONFIGS,
    KINDS,
    STACK_DENSE_HEADS,
    Config,
    DENSE,
    basis,
    basis_fp64,
    config,
    device_prompt_inputs,
    device_state,
    device_step_inputs,
    init_state,
    layer_rank_table,
    prompt_inputs,
    rank_table,
    stack_rank_tables,
    step_inputs,
)

"""Seeded synthetic workloads for the MTGR HSTU-block forward.

This package draws random numbers only. It holds none of the method's arithmetic
(no normalisation, projection, attention or mask logic), so that both the CPU
oracle and the CUDA path can take their inputs from it without sharing code.
"""

from .workloads import (  # noqa: F401
    WORKLOADS,
    Workload,
    make_lengths,
    make_timestamps,
    make_tokens,
    make_block_params,
    make_stack_params,
    make_rab_tables,
    make_qkvu,
    make_workload,
    assemble_workload,
    bf16_round,
    group_scales,
    sweep_expanded,
    TOKEN_F,
    HEAD_DH,
    N_TASKS,
    make_token_inputs,
    make_token_params,
    make_head_params,
)

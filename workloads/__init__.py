"""Seeded synthetic inputs for decode-time Multi-head Latent Attention.

This package only draws random numbers and rounds them to the storage
precision of a workload.  It holds none of the attention arithmetic, so both
the CPU oracle and the CUDA path can take their inputs from it without
sharing any computation.
"""

from .synth import (  # noqa: F401
    Workload,
    WORKLOADS,
    bf16_round,
    bf16_bits,
    draw_weights,
    draw_query_weights,
    ctx_lengths,
    block_table,
    hidden_states,
    queries,
    random_cache,
)

"""Seeded synthetic workloads for the OneTrans block stack.

This package only draws random numbers and lays them out in the shapes of the
workloads.  It holds none of the block's arithmetic (no norm, projection,
attention, pyramid schedule or quantisation), so the CPU oracle and the CUDA
path can both consume its output without sharing any of the method's code.
"""

from .workloads import (  # noqa: F401
    WORKLOADS,
    Workload,
    gen_auto_split_features,
    gen_embedding_table,
    gen_s_tokens,
    gen_weights,
    gen_zipf_ids,
    storage_round,
)

"""Seeded synthetic inputs for the Sparse-to-Dense (StD) decoding hot path.

This package holds no arithmetic of the method itself: it only draws the
tensors (queries, keys, values, token streams) that both the fp64 oracle and
the CUDA library consume, and rounds them to the storage type once so both
sides read identical bits.
"""
from .generator import (  # noqa: F401
    WORKLOADS,
    Workload,
    bf16_bits_to_f64,
    decode_kv,
    decode_queries,
    host_inputs,
    kv_head,
    planted,
    q_text_head,
    ragged_workload,
    storage,
    storage_to_f64,
    tokens,
    workload,
)

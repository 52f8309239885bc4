"""Seeded synthetic inputs shared by the oracle side and the CUDA side of the tests.

This package draws random numbers and rounds them to BF16; it holds none of the
FlashLoop method's arithmetic (no quantisation, reconstruction or attention).
"""
from .gen import (  # noqa: F401
    HEAD_DIM,
    GROUP,
    TAIL,
    Workload,
    WORKLOADS,
    active_sets,
    depth_of,
    prefill_layer,
    decode_token,
    hidden_states,
    queries,
    split_prefill,
)

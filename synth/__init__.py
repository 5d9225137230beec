"""Seeded synthetic inputs for PQ-HSA decode (shared by the tests, the bench and smoke).

This module draws random numbers and lays them out in the buffers both the CUDA
library and the CPU oracle consume. It holds none of the method's arithmetic:
no logits, no selection, no encoding, no attention.
"""
from .workloads import (  # noqa: F401
    Workload,
    WORKLOADS,
    workload,
    UnitData,
    Batch,
    make_batch,
    make_unit,
    f32_to_bf16_bits,
    bf16_bits_to_f32,
    train_init_slots,
)

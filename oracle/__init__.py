"""Plain float64 CPU oracle for PQ-HSA decode attention.

TEST INFRASTRUCTURE ONLY. Only the tests, the smoke entry and the bench's CPU
baseline leg may import this package; the library never does, and the library
shares no code with it.
"""
from .pqhsa_oracle import (  # noqa: F401
    widen_bf16,
    unit_rows,
    pq_lut,
    approx_logits,
    select_topk,
    cluster_means,
    decode_unit,
    dense_unit,
    encode_keys,
    oracle_decode,
    oracle_dense,
    oracle_build_means,
    oracle_append,
    decode_k,
    lloyd_assign,
    lloyd_update,
    kmeans_objective,
    train_unit,
    oracle_train,
)

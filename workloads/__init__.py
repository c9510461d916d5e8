"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle checks.

This package holds no attention arithmetic: it only draws random tensors,
rounds them to bf16 and builds index tables with the shapes, distributions and
sparsity structure of the workloads.  Both the CUDA library and the CPU oracle
consume what it returns; neither is imported here.
"""
from .gen import (  # noqa: F401
    Problem,
    WORKLOADS,
    bf16_round,
    bf16_bits,
    make_problem,
    make_fa_problem,
    make_device_problem,
    RowView,
    FAProblem,
    tiny_problem,
    subproblem,
    IndexerProblem,
    INDEXER_WORKLOAD,
    indexer_problem,
    make_device_indexer_problem,
)

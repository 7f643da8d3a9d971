"""Seeded synthetic workloads shared by the oracle tests, the GPU tests and the benchmark.

This package draws random numbers and lays them out; it holds none of the attention method's
arithmetic (no offsets, segment IDs, bounds, masks or softmax). Both the CPU oracle and the CUDA
path receive exactly the arrays produced here.
"""

from .workloads import (  # noqa: F401
    Batch,
    CandOnlyBatch,
    WORKLOADS,
    make_workload,
    tiny,
    three_users,
    users256,
    cand_only256,
    retrieval,
    custom_batch,
    custom_cand_only,
    users256_history_lengths,
    lognormal_history_lengths,
    users_batch,
    StackBatch,
    custom_stack,
    upstream_grad,
    stack_users256,
    UgBatch,
    custom_ug,
    ug_sep16k,
)

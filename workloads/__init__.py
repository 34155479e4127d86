"""Seeded synthetic workloads for tree speculative decoding verification.

This package only *generates inputs*: token trees given as ``parent[]``,
query / KV-cache tensors, target logits, speculative-model (SSM)
distributions and the uniform random numbers the stochastic verifier
consumes.  It holds none of the verification arithmetic (no attention, no
masks, no acceptance tests), so both the CPU oracle and the CUDA path can
draw their inputs from it without sharing any of the method's code.
"""

from .gen import (  # noqa: F401
    CONFIGS,
    WORKLOAD_NAMES,
    Workload,
    config_workload,
    random_workload,
    splitmix64_uniforms,
    tree_expansion,
    tree_levels,
    tree_merge_chains,
    tree_random,
    dfs_relabel,
)

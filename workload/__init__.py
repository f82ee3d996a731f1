"""Seeded synthetic workloads for the paged decode path.

This package only draws inputs: sequence lengths, which physical block each
logical block lands in, the copy pairs of forked sequences, the new token's
slot, token ids by position (for block hashing), and bf16 values for q, k_new,
v_new and the KV pools.  It computes none
of the path itself (no gather, score, softmax, merge, append or KV copy), so it
can feed both the CUDA path and the CPU oracle; neither of those is imported
here.
"""

from .configs import CONFIGS, WorkloadSpec, get_spec  # noqa: F401
from .gen import Workload, make_workload, rank_seed, token_ids  # noqa: F401

"""The five paged-decode workloads, as data.

Shapes follow the pages' running example (a Llama-3.2-1B-like bf16 GQA cache,
32 KiB of KV per token over 16 layers x 8 kv heads x 64 dims x K,V x 2 bytes;
ithelp.ithome.com.tw article 10405755, opening paragraph), many concurrent
sequences of unpredictable length, and B = 16 tokens per block ("只用了 8 格，
為什麼占了 12 格？", section 阿頁的辦法).  Every value is N(0, 1) rounded to
bf16; every length recipe is seeded.
"""

import math
from dataclasses import dataclass, field
from typing import Optional, Tuple


@dataclass(frozen=True)
class WorkloadSpec:
    key: str
    title: str
    num_layers: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    seed: int
    lengths: str                  # recipe name, see gen._draw_lengths
    pool_factor: float = 1.25     # physical blocks = ceil(factor * blocks in use)
    fixed_num_blocks: Optional[int] = None
    partition_tokens: int = 0     # 0 = library default
    shared_groups: int = 0        # groups of sequences sharing a prefix
    shared_group_size: int = 0
    shared_prefix: int = 0        # full-block part of the shared prefix
    block_size_sweep: Tuple[int, ...] = field(default_factory=tuple)

    @property
    def scale(self):
        return 1.0 / math.sqrt(self.head_dim)

    @property
    def group(self):
        return self.num_q_heads // self.num_kv_heads


CONFIGS = {
    "tiny": WorkloadSpec(
        key="tiny", title="Tiny paged decode: 4 seqs {7,9,1,16}, 8q/2kv, d64, B4, 32-block pool",
        num_layers=1, num_seqs=4, num_q_heads=8, num_kv_heads=2, head_dim=64, block_size=4,
        seed=1, lengths="fixed:7,9,1,16", fixed_num_blocks=32),
    "llama1b_layer": WorkloadSpec(
        key="llama1b_layer",
        title="Llama-3.2-1B-shaped layer: 64 seqs, len U[128,2048], 32q/8kv, d64, B16, append + attention",
        num_layers=1, num_seqs=64, num_q_heads=32, num_kv_heads=8, head_dim=64, block_size=16,
        seed=2, lengths="uniform:128,2048"),
    "continuous_batch": WorkloadSpec(
        key="continuous_batch",
        title="Continuous-batch mix: 256 seqs, len lognormal(median 300) in [1,4096], 32q/8kv, d64, B16, "
              "4 groups of 8 share a prefix and fork via copy-on-write",
        num_layers=1, num_seqs=256, num_q_heads=32, num_kv_heads=8, head_dim=64, block_size=16,
        seed=3, lengths="lognormal:300,1.0,1,4096",
        shared_groups=4, shared_group_size=8, shared_prefix=512),
    "long_context": WorkloadSpec(
        key="long_context",
        title="Long context split-K: 8 seqs x 32768, 32q/8kv, d128, B16, partitions of 512 tokens",
        num_layers=1, num_seqs=8, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
        seed=4, lengths="fixed_all:32768", partition_tokens=512),
    "full_step": WorkloadSpec(
        key="full_step",
        title="Full Llama-3.2-1B-shaped decode step: 16 layers x (append + attention), 512 seqs, "
              "len U[1,4096], 32q/8kv, d64, B in {8,16,32}",
        num_layers=16, num_seqs=512, num_q_heads=32, num_kv_heads=8, head_dim=64, block_size=16,
        seed=5, lengths="uniform:1,4096", block_size_sweep=(8, 16, 32)),
}

ORDER = ["tiny", "llama1b_layer", "continuous_batch", "long_context", "full_step"]


def get_spec(key):
    if key not in CONFIGS:
        raise KeyError(f"unknown workload {key!r}; known: {', '.join(ORDER)}")
    return CONFIGS[key]

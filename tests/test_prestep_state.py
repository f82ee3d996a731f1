"""Host logic of the bench's block-manager timing: the pre-step state it
derives from a workload, replayed through the oracle's BlockManager in the
workload's writer order, must give back the workload's own step (slots, copy
pairs, tables)."""

from collections import deque

import numpy as np
import pytest

import bench
from oracle.paging import BlockManager
from workload import make_workload


@pytest.mark.parametrize("key", ["tiny", "llama1b_layer", "continuous_batch", "full_step"])
def test_prestep_state_replays_to_the_workload_step(key):
    w = make_workload(key, values=False)
    st = bench.prestep_state(w)
    N, B = w.num_seqs, w.block_size
    bm = BlockManager(w.num_blocks, B)
    bm.free = deque(int(b) for b in st["free_ring"][:st["free_state"][1]])
    bm.refcount = [int(x) for x in st["refcount"]]
    for s in range(N):
        n = -(-int(st["seq_lens"][s]) // B)
        bm.tables[s] = [int(x) for x in st["block_tables"][s, :n]]
        bm.lengths[s] = int(st["seq_lens"][s])
    # every block is either free or used, never both
    used = {b for t in bm.tables.values() for b in t}
    assert used.isdisjoint(bm.free) and len(used) + len(bm.free) <= w.num_blocks
    slots = np.zeros(N, np.int64)
    for s in w.batch_order:
        slots[int(s)] = bm.append_slot(int(s))
    assert np.array_equal(slots, w.slot_mapping)
    assert np.array_equal(np.array(bm.take_copy_pairs(), np.int32).reshape(-1, 2), w.copy_pairs)
    for s in range(N):
        assert list(w.block_tables[s, :len(bm.tables[s])]) == bm.tables[s]


@pytest.mark.parametrize("key", ["continuous_batch", "tiny"])
def test_cow_sources_name_the_writers_that_copy(key):
    # replaying the step through the oracle, each sequence that copies its tail
    # does so from the block cow_sources gives it; every other sequence gets -1
    w = make_workload(key, values=False)
    st = bench.prestep_state(w)
    N, B = w.num_seqs, w.block_size
    bm = BlockManager(w.num_blocks, B)
    bm.free = deque(int(b) for b in st["free_ring"][:st["free_state"][1]])
    bm.refcount = [int(x) for x in st["refcount"]]
    for s in range(N):
        n = -(-int(st["seq_lens"][s]) // B)
        bm.tables[s] = [int(x) for x in st["block_tables"][s, :n]]
        bm.lengths[s] = int(st["seq_lens"][s])
    want = np.full(N, -1, np.int32)
    for s in w.batch_order:
        before = len(bm.copy_pairs)
        bm.append_slot(int(s))
        if len(bm.copy_pairs) > before:
            want[int(s)] = bm.copy_pairs[-1][0]
    assert np.array_equal(bench.cow_sources(w), want)

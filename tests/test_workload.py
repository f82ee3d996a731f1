"""The seeded generator against the oracle's pinned block manager.

Replaying each workload's allocation through ``oracle.paging.BlockManager``
(prefill, fork, append with copy-on-write) must give the same block tables,
new-token slots and copy pairs the generator wrote, so both sides of every
parity test are fed inputs that obey the pages' block rules.
"""

import numpy as np
import pytest

from oracle import paging as op
from workload import make_workload, rank_seed
from workload.configs import ORDER, get_spec


def _replay(w):
    spec = w.spec
    B = w.block_size
    bm = op.BlockManager(w.num_blocks, B, free_order=w.free_order.tolist())
    order = w.batch_order.tolist()
    gs = spec.shared_group_size
    n_shared = spec.shared_groups * gs
    slots = {}
    for g in range(spec.shared_groups):
        members = order[g * gs:(g + 1) * gs]
        leader = members[0]
        bm.add_sequence(leader, int(w.seq_lens[leader]) - 1)
        for m in members[1:]:
            bm.fork(leader, m)
        for m in members:
            slots[m] = bm.append_slot(m)
    for pos in order[n_shared:]:
        bm.add_sequence(pos, int(w.seq_lens[pos]) - 1)
        slots[pos] = bm.append_slot(pos)
    return bm, slots


@pytest.mark.parametrize("key,B", [(k, None) for k in ORDER] + [("full_step", 8), ("full_step", 32)])
def test_generator_agrees_with_block_manager(key, B):
    w = make_workload(key, block_size=B, values=False)
    bm, slots = _replay(w)
    for s in range(w.num_seqs):
        n = int(w.seq_lens[s])
        nb = op.blocks_needed(n, w.block_size)
        assert w.block_tables[s, :nb].tolist() == bm.tables[s]
        assert np.all(w.block_tables[s, nb:] == -1)
        assert int(w.slot_mapping[s]) == slots[s]
        assert int(w.slot_mapping[s]) == op.flat_slot(bm.tables[s], n - 1, w.block_size)
    assert [tuple(p) for p in w.copy_pairs.tolist()] == bm.take_copy_pairs()
    # every slot of the step is distinct
    assert len(set(w.slot_mapping.tolist())) == w.num_seqs


def test_shared_prefix_shape_of_the_continuous_batch_mix():
    w = make_workload("continuous_batch", values=False)
    spec = w.spec
    assert len(w.copy_pairs) == spec.shared_groups * (spec.shared_group_size - 1)
    dst = w.copy_pairs[:, 1]
    assert len(set(dst.tolist())) == len(dst)
    assert not set(dst.tolist()) & set(w.copy_pairs[:, 0].tolist())
    # a destination holds no live KV before the step; a source does
    assert not w.live_before[dst].any()
    assert w.live_before[w.copy_pairs[:, 0]].any(axis=1).all()
    lens = w.seq_lens
    assert 1 <= lens.min() and lens.max() <= 4096


def test_lengths_follow_the_recipes():
    w = make_workload("llama1b_layer", values=False)
    assert w.seq_lens.min() >= 128 and w.seq_lens.max() <= 2048
    w = make_workload("tiny", values=False)
    assert w.seq_lens.tolist() == [7, 9, 1, 16] and w.num_blocks == 32
    assert int((w.block_tables >= 0).sum()) == 10
    w = make_workload("long_context", values=False)
    assert np.all(w.seq_lens == 32768)


def test_values_are_seeded_and_poisoned():
    a = make_workload("tiny")
    b = make_workload("tiny")
    assert a.k_pool.equal(b.k_pool) or (a.k_pool.view(torch_int16()).equal(b.k_pool.view(torch_int16())))
    live = a.live_before
    bits = a.k_pool[0].view(torch_int16()).numpy().view(np.uint16)   # [NB, H, B, d]
    dead = ~live
    assert np.all(bits.transpose(0, 2, 1, 3)[dead] == 0x7FC0)
    assert not np.any(bits.transpose(0, 2, 1, 3)[live] == 0x7FC0)
    c = make_workload("tiny", seed=rank_seed(1, 1))
    assert not c.q.view(torch_int16()).equal(a.q.view(torch_int16()))


def torch_int16():
    import torch
    return torch.int16

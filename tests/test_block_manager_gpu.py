"""GPU parity of the device-side block manager step against the oracle's
pinned BlockManager (append_slot in writer order), on states built by the
oracle: tables, lengths, reference counts, the free ring, slot mapping and
copy pairs must all match exactly.
"""

import numpy as np
import pytest
import torch

from oracle.paging import BlockManager
from workload import make_workload

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import paged_kv_cache_378_b200 as pkv
else:  # collected on CPU-only machines, never run there
    pkv = None


@pytest.fixture(autouse=True)
def _clean_status():
    if torch.cuda.is_available():
        pkv.get_device_status(reset=True)
    yield


def _snapshot(bm, writers, max_blocks):
    """Device copy of the oracle's state; row i of the tables is writer sequence writers[i]."""
    N = len(writers)
    tables = np.full((N, max_blocks), -1, np.int32)
    for i, s in enumerate(writers):
        t = bm.tables[s]
        tables[i, :len(t)] = t
    lens = np.array([bm.lengths[s] for s in writers], np.int32)
    ring = np.full(bm.num_blocks, -1, np.int32)
    free = list(bm.free)
    ring[:len(free)] = free
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return pkv.BlockState(dev(tables), dev(lens), dev(np.array(bm.refcount, np.int32)), dev(ring),
                          dev(np.array([0, len(free)], np.int32)))


def _run_and_compare(bm, writers, max_blocks, order_rows, B):
    """Device step (rows in order_rows) against oracle append_slot in the same order."""
    st = _snapshot(bm, writers, max_blocks)
    order = torch.tensor(order_rows, dtype=torch.int32, device="cuda")
    slots, pairs, npairs = pkv.block_manager_step(st, B, order=order)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    want_slots = np.zeros(len(writers), np.int64)
    for i in order_rows:
        want_slots[i] = bm.append_slot(writers[i])
    want_pairs = np.array(bm.take_copy_pairs(), np.int32).reshape(-1, 2)
    n = int(npairs.item())
    assert n == len(want_pairs)
    assert np.array_equal(pairs[:n].cpu().numpy(), want_pairs)
    assert np.array_equal(slots.cpu().numpy(), want_slots)
    tab = st.block_tables.cpu().numpy()
    for i, s in enumerate(writers):
        t = bm.tables[s]
        assert list(tab[i, :len(t)]) == t, f"table of writer {i}"
    assert np.array_equal(st.seq_lens.cpu().numpy(), [bm.lengths[s] for s in writers])
    assert np.array_equal(st.refcount.cpu().numpy(), bm.refcount)
    head, count = st.free_state.cpu().numpy().tolist()
    ring = st.free_ring.cpu().numpy()
    assert count == len(bm.free)
    assert [int(ring[(head + k) % bm.num_blocks]) for k in range(count)] == list(bm.free)
    return slots, pairs[:n]


def test_page_example_new_block_when_tail_is_full():
    # ithelp 10405755, 手動畫一次 block table: B = 4, table [7, 1] holds 8 tokens;
    # the 9th token takes the free block 3 -> [7, 1, 3], slot 12
    bm = BlockManager(8, 4, free_order=[7, 1, 3, 0, 2, 4, 5, 6])
    bm.add_sequence("A", 8)
    slots, pairs = _run_and_compare(bm, ["A"], 4, [0], 4)
    assert slots.tolist() == [12] and len(pairs) == 0


def test_page_example_copy_on_write():
    # Infra: PagedAttention, 共享前缀，分叉时 Copy-on-write: A and B share [P3, P0] with
    # 6 tokens (B = 4); A writes first and copies P0 -> P4, B keeps P0
    bm = BlockManager(8, 4, free_order=[3, 0, 4, 1, 2, 5, 6, 7])
    bm.add_sequence("A", 6)
    bm.fork("A", "B")
    slots, pairs = _run_and_compare(bm, ["A", "B"], 4, [0, 1], 4)
    assert pairs.cpu().tolist() == [[0, 4]]
    assert slots.tolist() == [4 * 4 + 2, 0 * 4 + 2]


def test_sharers_not_all_writing_all_copy():
    # 8 sharers of a partial tail, only 5 write this step: each sees a count
    # above one, so all 5 copy and the block keeps 3 users
    bm = BlockManager(64, 16, free_order=np.random.default_rng(3).permutation(64))
    bm.add_sequence(0, 40)
    for c in range(1, 8):
        bm.fork(0, c)
    writers = [1, 3, 4, 6, 7]
    _run_and_compare(bm, writers, 8, [4, 0, 2, 1, 3], 16)
    assert bm.refcount[bm.tables[0][-1]] == 3


@pytest.mark.parametrize("N,B,seed", [(256, 16, 1), (512, 8, 2), (4096, 32, 3), (37, 4, 4)])
def test_random_batches_with_shared_prefixes(N, B, seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(1, 600, N)
    lens[rng.choice(N, N // 8, replace=False)] = rng.integers(1, 20, N // 8) * B   # full tails
    need = int(sum(-(-int(n) // B) for n in lens)) + N + 8 * 51 + 64
    NB = int(need * 1.25)
    bm = BlockManager(NB, B, free_order=rng.permutation(NB))
    # groups of 8 sharing a prefix with a partial tail, the rest independent
    groups = min(8, N // 8)
    writers = []
    for g in range(groups):
        root = ("g", g)
        bm.add_sequence(root, int(rng.integers(2, 50)) * B + int(rng.integers(1, B)))
        writers.append(root)
        for c in range(7):
            bm.fork(root, ("c", g, c))
            writers.append(("c", g, c))
    for i in range(N - len(writers)):
        bm.add_sequence(("s", i), int(lens[i]))
        writers.append(("s", i))
    max_blocks = max(len(t) for t in bm.tables.values()) + 2
    _run_and_compare(bm, writers, max_blocks, rng.permutation(N).tolist(), B)


def test_out_of_blocks_changes_nothing():
    bm = BlockManager(6, 4, free_order=range(6))
    for s in range(3):
        bm.add_sequence(s, 4)          # full tails: each writer needs a block, 3 free
    bm.add_sequence(3, 3)              # 4 blocks used, 2 free
    st = _snapshot(bm, [0, 1, 2, 3], 4)
    before = [t.clone() for t in (st.block_tables, st.seq_lens, st.refcount, st.free_ring,
                                  st.free_state)]
    pkv.block_manager_step(st, 4)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == pkv.DEV_NOBLOCKS
    after = (st.block_tables, st.seq_lens, st.refcount, st.free_ring, st.free_state)
    for a, b in zip(before, after):
        assert torch.equal(a, b)


def test_step_then_copy_then_fused_attention_runs_on_device_counts():
    # the whole decode step with no host round trip: manager -> block copy with the
    # device-side pair count -> fused append + attention; pools checked against
    # the same step driven from the oracle's slot mapping and pairs
    from oracle import attention as oa
    from .stepping import assert_close, f64, u16
    rng = np.random.default_rng(7)
    B, H, D, G, NB = 16, 2, 64, 4, 96
    bm = BlockManager(NB, B, free_order=rng.permutation(NB))
    bm.add_sequence(0, 37)
    for c in range(1, 4):
        bm.fork(0, c)
    for s in range(4, 10):
        bm.add_sequence(s, int(rng.integers(1, 70)))
    writers = list(range(10))
    st = _snapshot(bm, writers, 8)
    g = torch.Generator().manual_seed(7)
    kp = torch.randn((1, NB, H, B, D), generator=g).to(torch.bfloat16)
    vp = torch.randn((1, NB, H, B, D), generator=g).to(torch.bfloat16)
    q = torch.randn((10, H * G, D), generator=g).to(torch.bfloat16)
    kn = torch.randn((10, H, D), generator=g).to(torch.bfloat16)
    vn = torch.randn((10, H, D), generator=g).to(torch.bfloat16)
    kd, vd = kp.cuda(), vp.cuda()
    slots, pairs, npairs = pkv.block_manager_step(st, B)
    pkv.block_copy(pairs, kd, vd, num_pairs=npairs)
    out = torch.empty_like(q).cuda()
    ws = pkv.make_workspace(10, H * G, H, D, 8, B, 0)
    pkv.append_paged_decode_attention(kn.cuda(), vn.cuda(), q.cuda(), kd, vd, st.block_tables,
                                      st.seq_lens, B, D ** -0.5, out, workspace=ws)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    want_slots = [bm.append_slot(s) for s in writers]
    want_pairs = np.array(bm.take_copy_pairs(), np.int32).reshape(-1, 2)
    assert slots.cpu().tolist() == want_slots
    ek, ev = oa.block_copy(u16(kp), u16(vp), want_pairs)
    ek, ev = oa.kv_append(ek[0], ev[0], u16(kn), u16(vn), np.array(want_slots), B)
    assert np.array_equal(u16(kd[0]), ek) and np.array_equal(u16(vd[0]), ev)
    tables = np.full((10, 8), -1, np.int32)
    for s in writers:
        tables[s, :len(bm.tables[s])] = bm.tables[s]
    lens = np.array([bm.lengths[s] for s in writers], np.int32)
    ref = oa.paged_decode_attention(u16(q), ek, ev, tables, lens, B, D ** -0.5)
    assert_close(f64(out), ref, "device-managed step")


@pytest.mark.parametrize("key,B", [("tiny", None), ("llama1b_layer", None),
                                   ("continuous_batch", None), ("full_step", 8),
                                   ("full_step", 16), ("full_step", 32)])
def test_workload_steps_at_full_size(key, B):
    # the device step on each workload's pre-step state, in its writer order,
    # reproduces the workload's own slots, copy pairs and tables (the generator
    # is pinned to the oracle's BlockManager on the CPU)
    import bench
    w = make_workload(key, block_size=B, values=False)
    st_np = bench.prestep_state(w)
    st = pkv.BlockState(**{k: torch.from_numpy(v).cuda() for k, v in st_np.items()})
    order = torch.from_numpy(np.ascontiguousarray(w.batch_order, dtype=np.int32)).cuda()
    slots, pairs, npairs = pkv.block_manager_step(st, w.block_size, order=order)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    n = int(npairs.item())
    assert np.array_equal(slots.cpu().numpy(), w.slot_mapping)
    assert np.array_equal(pairs[:n].cpu().numpy(), w.copy_pairs)
    assert np.array_equal(st.seq_lens.cpu().numpy(), w.seq_lens)
    tab = st.block_tables.cpu().numpy()
    for s in range(w.num_seqs):
        nb = -(-int(w.seq_lens[s]) // w.block_size)
        assert np.array_equal(tab[s, :nb], w.block_tables[s, :nb])


def test_device_step_with_copy_on_write_folded_into_attention():
    # manager -> one fused launch that copies the shared tails, appends and
    # attends: pools equal the oracle's block copy + append, output within
    # tolerance of the oracle
    from oracle import attention as oa
    from .stepping import assert_close, f64, u16
    rng = np.random.default_rng(11)
    B, H, D, G, NB = 16, 2, 64, 4, 120
    bm = BlockManager(NB, B, free_order=rng.permutation(NB))
    bm.add_sequence(0, 45)
    for c in range(1, 5):
        bm.fork(0, c)
    for s in range(5, 12):
        bm.add_sequence(s, int(rng.integers(1, 90)))
    writers = list(range(12))
    st = _snapshot(bm, writers, 8)
    g = torch.Generator().manual_seed(11)
    kp = torch.randn((1, NB, H, B, D), generator=g).to(torch.bfloat16)
    vp = torch.randn((1, NB, H, B, D), generator=g).to(torch.bfloat16)
    q = torch.randn((12, H * G, D), generator=g).to(torch.bfloat16)
    kn = torch.randn((12, H, D), generator=g).to(torch.bfloat16)
    vn = torch.randn((12, H, D), generator=g).to(torch.bfloat16)
    kd, vd = kp.cuda(), vp.cuda()
    slots, pairs, npairs, cow = pkv.block_manager_step(st, B, with_cow_src=True)
    out = torch.empty_like(q).cuda()
    ws = pkv.make_workspace(12, H * G, H, D, 8, B, 0)
    pkv.append_paged_decode_attention(kn.cuda(), vn.cuda(), q.cuda(), kd, vd, st.block_tables,
                                      st.seq_lens, B, D ** -0.5, out, workspace=ws, cow_src=cow)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    want_slots = [bm.append_slot(s) for s in writers]
    want_pairs = np.array(bm.take_copy_pairs(), np.int32).reshape(-1, 2)
    assert len(want_pairs) == 4 and int(npairs.item()) == 4
    assert slots.cpu().tolist() == want_slots
    ek, ev = oa.block_copy(u16(kp), u16(vp), want_pairs)
    ek, ev = oa.kv_append(ek[0], ev[0], u16(kn), u16(vn), np.array(want_slots), B)
    assert np.array_equal(u16(kd[0]), ek) and np.array_equal(u16(vd[0]), ev)
    tables = np.full((12, 8), -1, np.int32)
    for s in writers:
        tables[s, :len(bm.tables[s])] = bm.tables[s]
    lens = np.array([bm.lengths[s] for s in writers], np.int32)
    ref = oa.paged_decode_attention(u16(q), ek, ev, tables, lens, B, D ** -0.5)
    assert_close(f64(out), ref, "copy-on-write folded into attention")


def test_aborted_step_leaves_a_chained_device_step_harmless():
    # Free blocks run short: the manager changes no state and writes outputs
    # that make what is already queued behind it do nothing -- slots -1, no
    # copy pair, cow_src = COW_NO_APPEND -- so a device-only step chained on
    # the same stream (block copy with the device count, kv_append, fused
    # append + attention with cow_src) leaves both pools byte-identical.
    from .stepping import u16
    rng = np.random.default_rng(5)
    B, H, D, G, NB = 16, 2, 64, 4, 16
    bm = BlockManager(NB, B, free_order=rng.permutation(NB))
    bm.add_sequence(0, 37)             # 3 blocks, shared tail below: 3 copies needed
    for c in range(1, 4):
        bm.fork(0, c)
    for s in range(4, 8):
        bm.add_sequence(s, 32)         # full tails: 4 more blocks needed
    assert len(bm.free) == 5           # 7 needed
    writers = list(range(8))
    st = _snapshot(bm, writers, 4)
    before = [t.clone() for t in (st.block_tables, st.seq_lens, st.refcount, st.free_ring,
                                  st.free_state)]
    g = torch.Generator().manual_seed(5)
    kd = torch.randn((1, NB, H, B, D), generator=g).to(torch.bfloat16).cuda()
    vd = torch.randn((1, NB, H, B, D), generator=g).to(torch.bfloat16).cuda()
    k0, v0 = u16(kd), u16(vd)
    q = torch.randn((8, H * G, D), generator=g).to(torch.bfloat16).cuda()
    kn = torch.randn((8, H, D), generator=g).to(torch.bfloat16).cuda()
    vn = torch.randn((8, H, D), generator=g).to(torch.bfloat16).cuda()
    slots, pairs, npairs, cow = pkv.block_manager_step(st, B, with_cow_src=True)
    pkv.block_copy(pairs, kd, vd, num_pairs=npairs)
    pkv.kv_append(kn, vn, slots, kd, vd)
    out = torch.empty_like(q)
    ws = pkv.make_workspace(8, H * G, H, D, 4, B, 0)
    pkv.append_paged_decode_attention(kn, vn, q, kd, vd, st.block_tables, st.seq_lens, B,
                                      D ** -0.5, out, workspace=ws, cow_src=cow)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == pkv.DEV_NOBLOCKS
    assert slots.cpu().tolist() == [-1] * 8
    assert int(npairs.item()) == 0
    assert cow.cpu().tolist() == [pkv.COW_NO_APPEND] * 8
    assert np.array_equal(u16(kd), k0) and np.array_equal(u16(vd), v0)
    after = (st.block_tables, st.seq_lens, st.refcount, st.free_ring, st.free_state)
    for a, b in zip(before, after):
        assert torch.equal(a, b)

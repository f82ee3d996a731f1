"""GPU parity of the device-side release of finished requests against the
oracle's pinned BlockManager.free_sequence: rows released in the given order
drop one reference per block in table order, blocks left without users join
the free ring in that order, the rows' lengths become 0 and their tables -1.
Reference counts and the whole free ring (order included) must match exactly.
"""

import numpy as np
import pytest
import torch

from oracle.paging import BlockManager

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


def _snapshot(bm, rows, max_blocks):
    """Device copy of the oracle's state; row i holds sequence rows[i]."""
    N = len(rows)
    tables = np.full((N, max_blocks), -1, np.int32)
    for i, s in enumerate(rows):
        t = bm.tables[s]
        tables[i, :len(t)] = t
    lens = np.array([bm.lengths[s] for s in rows], np.int32)
    ring = np.full(bm.num_blocks, -1, np.int32)
    free = list(bm.free)
    ring[:len(free)] = free
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return pkv.BlockState(dev(tables), dev(lens), dev(np.array(bm.refcount, np.int32)), dev(ring),
                          dev(np.array([0, len(free)], np.int32)))


def _release_and_compare(bm, rows, max_blocks, release_rows, B):
    st = _snapshot(bm, rows, max_blocks)
    seqs = torch.tensor(release_rows, dtype=torch.int32, device="cuda")
    pkv.block_manager_release(st, B, seqs)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    for i in release_rows:
        bm.free_sequence(rows[i])
    tab = st.block_tables.cpu().numpy()
    lens = st.seq_lens.cpu().numpy()
    for i, s in enumerate(rows):
        if i in release_rows:
            assert (tab[i] == -1).all() and lens[i] == 0, f"released row {i}"
        else:
            t = bm.tables[s]
            assert list(tab[i, :len(t)]) == t and lens[i] == bm.lengths[s], f"row {i}"
    assert np.array_equal(st.refcount.cpu().numpy(), bm.refcount)
    head, count = st.free_state.cpu().numpy().tolist()
    ring = st.free_ring.cpu().numpy()
    assert head == 0 and count == len(bm.free)
    assert [int(ring[(head + k) % bm.num_blocks]) for k in range(count)] == list(bm.free)
    return st


def test_page_example_request_end_returns_its_blocks():
    # ithelp 10405755, 手動畫一次 block table: A ends holding [7, 1, 3] (9 tokens,
    # B = 4); the three blocks go back to the pool, after the free ones
    bm = BlockManager(8, 4, free_order=[7, 1, 3, 0, 2, 4, 5, 6])
    bm.add_sequence("A", 9)
    bm.add_sequence("B", 2)
    assert bm.tables["A"] == [7, 1, 3]
    _release_and_compare(bm, ["A", "B"], 4, [0], 4)
    assert list(bm.free)[-3:] == [7, 1, 3]


def test_shared_blocks_return_only_with_their_last_user():
    # Infra: PagedAttention, 共享前缀，分叉时 Copy-on-write: A and B share [P3, P0];
    # after A copied P0 -> P4, releasing A frees only P4, releasing B then frees P3, P0
    bm = BlockManager(8, 4, free_order=[3, 0, 4, 1, 2, 5, 6, 7])
    bm.add_sequence("A", 6)
    bm.fork("A", "B")
    bm.append_slot("A")
    bm.append_slot("B")
    bm.take_copy_pairs()
    rows = ["A", "B"]
    bm2 = BlockManager(8, 4, free_order=[3, 0, 4, 1, 2, 5, 6, 7])
    bm2.add_sequence("A", 6)
    bm2.fork("A", "B")
    bm2.append_slot("A")
    bm2.append_slot("B")
    _release_and_compare(bm, rows, 4, [0], 4)                 # A alone
    assert list(bm.free)[-1:] == [4]
    _release_and_compare(bm2, rows, 4, [1, 0], 4)             # both in one call, B first
    assert list(bm2.free)[-3:] == [0, 3, 4]                 # 0 at B's last drop, then 3 and 4


@pytest.mark.parametrize("N,B,seed", [(256, 16, 1), (512, 8, 2), (4096, 32, 3), (37, 4, 4)])
def test_random_releases_with_shared_prefixes(N, B, seed):
    rng = np.random.default_rng(seed)
    lens = rng.integers(0, 600, N)
    need = int(sum(-(-int(n) // B) for n in lens)) + 8 * 51 + 64
    NB = int(need * 1.25)
    bm = BlockManager(NB, B, free_order=rng.permutation(NB))
    groups = min(8, N // 8)
    rows = []
    for g in range(groups):
        root = ("g", g)
        bm.add_sequence(root, int(rng.integers(2, 50)) * B + int(rng.integers(0, B)))
        rows.append(root)
        for c in range(7):
            bm.fork(root, ("c", g, c))
            rows.append(("c", g, c))
    for i in range(N - len(rows)):
        bm.add_sequence(("s", i), int(lens[i]))
        rows.append(("s", i))
    # some sharers write a token (copy-on-write), so tables differ in their tails
    for i in rng.choice(len(rows), len(rows) // 4, replace=False):
        bm.append_slot(rows[int(i)])
    bm.take_copy_pairs()
    max_blocks = max(len(t) for t in bm.tables.values()) + 1
    release = rng.choice(N, N // 3, replace=False).tolist()
    _release_and_compare(bm, rows, max_blocks, release, B)


def test_released_row_takes_a_fresh_block_on_the_next_step():
    # a released row serves a new request: the step gives it a block for token 0
    bm = BlockManager(16, 4, free_order=np.random.default_rng(5).permutation(16))
    bm.add_sequence(0, 7)
    bm.add_sequence(1, 5)
    st = _release_and_compare(bm, [0, 1], 4, [0], 4)
    slots, pairs, npairs = pkv.block_manager_step(st, 4)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    bm.add_sequence(0, 0)
    want = [bm.append_slot(0), bm.append_slot(1)]
    assert slots.cpu().tolist() == want and int(npairs.item()) == 0
    assert st.block_tables.cpu().numpy()[0, 0] == bm.tables[0][0]
    assert st.seq_lens.cpu().tolist() == [1, 6]


@pytest.mark.parametrize("bad", ["twice", "out_of_range"])
def test_invalid_release_changes_nothing(bad):
    bm = BlockManager(16, 4, free_order=range(16))
    for s in range(3):
        bm.add_sequence(s, 5)
    st = _snapshot(bm, [0, 1, 2], 4)
    before = [t.clone() for t in (st.block_tables, st.seq_lens, st.refcount, st.free_ring,
                                  st.free_state)]
    rows = [1, 0, 1] if bad == "twice" else [0, 3]
    pkv.block_manager_release(st, 4, torch.tensor(rows, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == pkv.DEV_RANGE
    after = (st.block_tables, st.seq_lens, st.refcount, st.free_ring, st.free_state)
    for a, b in zip(before, after):
        assert torch.equal(a, b)

"""A device-resident continuous-batching loop against the oracle.

Every step the device block manager serves one new token per sequence
(copy-on-write of shared tails included) and, with no host read in between,
the fused launch copies the shared tails, appends the new tokens and attends.
Every few steps some requests finish: their rows release their blocks on the
device and start new requests (length 0, a fresh block on the next step).
After every step the device block state equals the oracle BlockManager's
(tables, lengths, counts, the free ring in order), the pools equal the
oracle's block copies + appends bit for bit, and the attention output is
within the tolerance of the oracle's.
"""

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle.paging import BlockManager

from .stepping import assert_close, f64, u16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import paged_kv_cache_378_b200 as pkv
else:  # collected on CPU-only machines, never run there
    pkv = None


def _state_arrays(bm, rows, max_blocks):
    tables = np.full((len(rows), max_blocks), -1, np.int32)
    for i, s in enumerate(rows):
        t = bm.tables[s]
        tables[i, :len(t)] = t
    lens = np.array([bm.lengths[s] for s in rows], np.int32)
    return tables, lens


def _device_state(bm, rows, max_blocks):
    tables, lens = _state_arrays(bm, rows, max_blocks)
    ring = np.full(bm.num_blocks, -1, np.int32)
    free = list(bm.free)
    ring[:len(free)] = free
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return pkv.BlockState(dev(tables), dev(lens), dev(np.array(bm.refcount, np.int32)), dev(ring),
                          dev(np.array([0, len(free)], np.int32)))


def _assert_state(st, bm, rows, max_blocks, what):
    tables, lens = _state_arrays(bm, rows, max_blocks)
    assert np.array_equal(st.block_tables.cpu().numpy(), tables), f"{what}: tables"
    assert np.array_equal(st.seq_lens.cpu().numpy(), lens), f"{what}: lengths"
    assert np.array_equal(st.refcount.cpu().numpy(), bm.refcount), f"{what}: counts"
    head, count = st.free_state.cpu().numpy().tolist()
    ring = st.free_ring.cpu().numpy()
    assert count == len(bm.free), f"{what}: free count"
    assert [int(ring[(head + k) % bm.num_blocks]) for k in range(count)] == list(bm.free), \
        f"{what}: free ring"


@pytest.mark.parametrize("B", [4, 16])
def test_device_loop_with_forks_and_releases(B):
    rng = np.random.default_rng(11 + B)
    gen = torch.Generator().manual_seed(11 + B)
    N, Hkv, G, D, steps = 12, 2, 2, 64, 24
    NB = 12 * (-(-(40 + steps) // B) + 2) + 16
    max_blocks = -(-(40 + steps) // B) + 1
    scale = D ** -0.5
    bm = BlockManager(NB, B, free_order=rng.permutation(NB))
    rows = list(range(N))
    # rows 0..3 share a prompt whose tail is partial (they copy on their first
    # write); the rest have independent prompts, some empty
    bm.add_sequence(0, 2 * B + 1)
    for c in (1, 2, 3):
        bm.fork(0, c)
    for s in range(4, N):
        bm.add_sequence(s, int(rng.integers(0, 40)))
    st = _device_state(bm, rows, max_blocks)
    k_pool = torch.randn((1, NB, Hkv, B, D), generator=gen).to(torch.bfloat16)
    v_pool = torch.randn((1, NB, Hkv, B, D), generator=gen).to(torch.bfloat16)
    dk, dv = k_pool.cuda(), v_pool.cuda()
    hk, hv = u16(k_pool[0]), u16(v_pool[0])
    ws = pkv.make_workspace(N, Hkv * G, Hkv, D, max_blocks, B, 0, device=torch.device("cuda"))
    pkv.get_device_status(reset=True)
    releases = 0
    for t in range(steps):
        q = torch.randn((N, Hkv * G, D), generator=gen).to(torch.bfloat16)
        k_new = torch.randn((N, Hkv, D), generator=gen).to(torch.bfloat16)
        v_new = torch.randn((N, Hkv, D), generator=gen).to(torch.bfloat16)
        out = torch.full((N, Hkv * G, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        # the device step: manager, then the fused launch on its outputs
        slots, pairs, npairs, cow = pkv.block_manager_step(st, B, with_cow_src=True)
        pkv.append_paged_decode_attention(k_new.cuda(), v_new.cuda(), q.cuda(), dk, dv,
                                          st.block_tables, st.seq_lens, B, scale, out,
                                          workspace=ws, cow_src=cow)
        # the oracle step
        want_slots = [bm.append_slot(s) for s in rows]
        want_pairs = bm.take_copy_pairs()
        kp, vp = oa.block_copy(hk[None], hv[None], np.array(want_pairs, np.int64).reshape(-1, 2))
        hk, hv = oa.kv_append(kp[0], vp[0], u16(k_new), u16(v_new), want_slots, B)
        tables, lens = _state_arrays(bm, rows, max_blocks)
        ref = oa.paged_decode_attention(u16(q), hk, hv, tables, lens, B, scale)
        torch.cuda.synchronize()
        assert pkv.get_device_status(reset=True) == 0, f"step {t}"
        assert slots.cpu().tolist() == want_slots, f"step {t}: slots"
        n = int(npairs.item())
        assert pairs[:n].cpu().tolist() == [list(p) for p in want_pairs], f"step {t}: copy pairs"
        _assert_state(st, bm, rows, max_blocks, f"step {t}")
        assert np.array_equal(u16(dk[0]), hk) and np.array_equal(u16(dv[0]), hv), f"step {t}: pools"
        assert_close(f64(out), ref, f"step {t}")
        # requests finish: release on the device, their rows start new ones
        if t % 6 == 5:
            done = rng.choice(N, 3, replace=False).tolist()
            pkv.block_manager_release(st, B, torch.tensor(done, dtype=torch.int32, device="cuda"))
            for s in done:
                bm.free_sequence(rows[s])
                bm.add_sequence(rows[s], 0)
            torch.cuda.synchronize()
            assert pkv.get_device_status(reset=True) == 0, f"release after step {t}"
            _assert_state(st, bm, rows, max_blocks, f"release after step {t}")
            releases += 1
    assert releases >= 3

"""GPU parity of the prefix-cache block hashes against the oracle (bit exact),
and the sharing property on workloads with shared prompts."""

import numpy as np
import pytest
import torch

from oracle import prefix_hash as ph
from workload import make_workload, token_ids

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


def _u64(x):
    return int(x) & ((1 << 64) - 1)


def _check(tokens, lens, B, keys, rows):
    got = pkv.prefix_block_hashes(torch.from_numpy(tokens).cuda(), torch.from_numpy(lens).cuda(), B,
                                  None if keys is None else torch.from_numpy(keys).cuda())
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    got = got.cpu().numpy()
    for s in rows:
        want = ph.prefix_block_hashes(tokens[s].tolist(), int(lens[s]), B,
                                      0 if keys is None else _u64(keys[s]))
        assert [_u64(x) for x in got[s, :len(want)]] == want, f"sequence {s}"
        assert not got[s, len(want):].any()
    return got


@pytest.mark.parametrize("B", [4, 8, 16, 32])
def test_random_sequences_with_keys(B):
    rng = np.random.default_rng(B)
    N, T = 70, 40 * B
    tokens = rng.integers(-2**31, 2**31 - 1, (N, T), dtype=np.int64).astype(np.int32)
    lens = rng.integers(0, T + 1, N).astype(np.int32)
    lens[:3] = [0, B - 1, B]
    keys = rng.integers(-2**63, 2**63 - 1, N, dtype=np.int64)
    _check(tokens, lens, B, keys, range(N))
    _check(tokens, lens, B, None, range(0, N, 7))


def test_continuous_batch_shared_prompts_hash_alike():
    w = make_workload("continuous_batch", values=False)
    tokens = token_ids(w)
    got = _check(tokens, w.seq_lens, w.block_size, None, range(w.num_seqs))
    # full blocks at the same logical index that are one physical block (a
    # shared prompt) have one hash
    B = w.block_size
    seen = {}
    shared = 0
    for s in range(w.num_seqs):
        for b in range(int(w.seq_lens[s]) // B):
            key = (b, int(w.block_tables[s, b]))
            if key in seen:
                assert seen[key] == got[s, b]
                shared += 1
            seen[key] = got[s, b]
    assert shared > 0


def test_full_step_sampled():
    w = make_workload("full_step", values=False)
    tokens = token_ids(w)
    rng = np.random.default_rng(5)
    _check(tokens, w.seq_lens, w.block_size, None, rng.choice(w.num_seqs, 12, replace=False))


def test_resume_from_a_parent_hash():
    # hashing from block k with the stored hash of block k-1 gives the same
    # hashes as hashing the whole prefix; blocks before k are left untouched
    # (the decode case: only the block that just became full)
    rng = np.random.default_rng(9)
    N, B, T = 50, 16, 640
    tokens = rng.integers(0, 128256, (N, T)).astype(np.int32)
    lens = rng.integers(0, T + 1, N).astype(np.int32)
    tok_d, len_d = torch.from_numpy(tokens).cuda(), torch.from_numpy(lens).cuda()
    whole = pkv.prefix_block_hashes(tok_d, len_d, B).cpu().numpy()
    nfull = lens // B
    first = np.array([rng.integers(0, n + 1) for n in nfull], np.int32)
    first[:4] = [0, nfull[1], max(nfull[2] - 1, 0), nfull[3]]
    parents = np.array([whole[s, first[s] - 1] if first[s] > 0 else 0 for s in range(N)], np.int64)
    out = torch.full((N, T // B), 7, dtype=torch.int64, device="cuda")
    res = pkv.prefix_block_hashes(tok_d, len_d, B, first_block=torch.from_numpy(first).cuda(),
                                  parent_hashes=torch.from_numpy(parents).cuda(), out=out)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    res = res.cpu().numpy()
    for s in range(N):
        assert np.array_equal(res[s, first[s]:nfull[s]], whole[s, first[s]:nfull[s]]), s
        assert np.all(res[s, :first[s]] == 7) and np.all(res[s, nfull[s]:] == 7), s
        want = ph.prefix_block_hashes(tokens[s].tolist(), int(lens[s]), B)
        assert [_u64(x) for x in res[s, first[s]:nfull[s]]] == want[first[s]:], s

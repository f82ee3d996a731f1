"""GPU parity: the CUDA path (through the C ABI binding) against the CPU oracle
on the same seeded inputs.

Bars: kv_append and block_copy bit exact (whole pools compared as uint16, NaN
poison included); attention elementwise |gpu - oracle| <= 1e-2 + 1e-2 |oracle|
(bf16 inputs, fp32 accumulation, bf16 output).
"""

import dataclasses

import numpy as np
import pytest
import torch

from oracle import attention as oa
from oracle import bf16 as ob
from workload import make_workload
from workload.configs import WorkloadSpec, get_spec

from .stepping import assert_close, device_inputs, f64, gpu_step, oracle_pools_after_step, u16

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


def _assert_no_device_error():
    assert pkv.get_device_status(reset=True) == 0


# ---------------------------------------------------------------------------
# kv_append / block_copy: bit exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("key", ["tiny", "llama1b_layer", "continuous_batch"])
def test_cow_copy_and_append_bit_exact(key):
    w = make_workload(key)
    dev = device_inputs(w)
    pkv.block_copy(dev["pairs"], dev["k_pool"], dev["v_pool"])
    pkv.kv_append(dev["k_new"][0], dev["v_new"][0], dev["slots"], dev["k_pool"], dev["v_pool"], layer=0)
    torch.cuda.synchronize()
    kp, vp = oracle_pools_after_step(w, u16(w.k_pool[0]), u16(w.v_pool[0]), 0)
    assert np.array_equal(u16(dev["k_pool"][0]), kp)
    assert np.array_equal(u16(dev["v_pool"][0]), vp)
    _assert_no_device_error()


def test_block_copy_every_layer_bit_exact():
    L, NB, H, B, d = 3, 64, 8, 16, 64
    g = torch.Generator().manual_seed(11)
    kp = torch.randn((L, NB, H, B, d), generator=g).to(torch.bfloat16)
    vp = torch.randn((L, NB, H, B, d), generator=g).to(torch.bfloat16)
    # odd bit patterns must survive: NaN payload, -0, denormal
    kp.view(torch.int16)[0, 5, 0, 0, :3] = torch.tensor([0x7FC1, -32768, 0x0001], dtype=torch.int16)
    pairs = np.array([[5, 40], [6, 41], [7, 63], [0, 1]], dtype=np.int32)
    kd, vd = kp.cuda(), vp.cuda()
    pkv.block_copy(torch.from_numpy(pairs).cuda(), kd, vd)
    torch.cuda.synchronize()
    ek, ev = oa.block_copy(u16(kp), u16(vp), pairs)
    assert np.array_equal(u16(kd), ek) and np.array_equal(u16(vd), ev)
    _assert_no_device_error()


def test_append_skips_padding_and_reports_bad_slots():
    NB, H, B, d = 8, 2, 8, 64
    kp = torch.zeros((NB, H, B, d), dtype=torch.bfloat16, device="cuda")
    vp = torch.zeros_like(kp)
    k = torch.randn((3, H, d), device="cuda").to(torch.bfloat16)
    v = torch.randn((3, H, d), device="cuda").to(torch.bfloat16)
    slots = torch.tensor([3, -1, NB * B + 5], dtype=torch.int64, device="cuda")
    pkv.kv_append(k, v, slots, kp, vp)
    assert pkv.get_device_status(reset=True) & pkv.DEV_RANGE
    ek, ev = oa.kv_append(u16(torch.zeros_like(kp)), u16(torch.zeros_like(vp)), u16(k[:1]),
                          u16(v[:1]), [3], B)
    assert np.array_equal(u16(kp), ek) and np.array_equal(u16(vp), ev)


# ---------------------------------------------------------------------------
# attention against the oracle
# ---------------------------------------------------------------------------

def _oracle_attention(w, layer, host_k=None, host_v=None):
    host_k = u16(w.k_pool[layer]) if host_k is None else host_k
    host_v = u16(w.v_pool[layer]) if host_v is None else host_v
    kp, vp = oracle_pools_after_step(w, host_k, host_v, layer)
    return oa.paged_decode_attention(u16(w.q[layer]), kp, vp, w.block_tables, w.seq_lens,
                                     w.block_size, w.spec.scale)


@pytest.mark.parametrize("key", ["tiny", "llama1b_layer", "continuous_batch"])
def test_attention_step_matches_oracle(key):
    w = make_workload(key)
    outs = gpu_step(pkv, w, device_inputs(w))
    _assert_no_device_error()
    ref = _oracle_attention(w, 0)
    assert_close(f64(outs[0]), ref, key)


@pytest.mark.parametrize("partition", [512, 2048, 0])
def test_long_context_split_k_matches_oracle(partition):
    w = make_workload("long_context")
    outs = gpu_step(pkv, w, device_inputs(w), partition_tokens=partition)
    _assert_no_device_error()
    ref = _oracle_attention(w, 0)
    assert_close(f64(outs[0]), ref, f"long_context partition={partition}")


@pytest.mark.parametrize("block_size", [8, 16, 32])
def test_full_step_first_and_last_layer_every_output(block_size):
    """Full 16-layer step at full size (512 sequences, lengths up to 4096);
    every output of the first and the last layer (512 x 32 heads) is compared
    with the oracle element by element (host copies of those layers' pools
    are taken before any kernel runs)."""
    w = make_workload("full_step", block_size=block_size, device="cuda")
    layers = [0, w.spec.num_layers - 1]
    host = {l: (u16(w.k_pool[l]), u16(w.v_pool[l])) for l in layers}
    dev = dict(k_pool=w.k_pool, v_pool=w.v_pool, q=w.q, k_new=w.k_new, v_new=w.v_new,
               tables=torch.from_numpy(w.block_tables).cuda(),
               lens=torch.from_numpy(w.seq_lens).cuda(),
               slots=torch.from_numpy(w.slot_mapping).cuda(),
               pairs=torch.from_numpy(w.copy_pairs).cuda())
    # the bench's step: one launch per layer doing copy-on-write, append, attention
    outs = gpu_step(pkv, w, dev, fused=True, cow=True)
    _assert_no_device_error()
    got = {l: f64(outs[l]) for l in layers}
    q = {l: u16(w.q[l]) for l in layers}
    tables, lens = w.block_tables, w.seq_lens
    B, scale = w.block_size, w.spec.scale
    del dev, outs
    w.k_pool = w.v_pool = None
    torch.cuda.empty_cache()
    for l in layers:
        kp, vp = oracle_pools_after_step(w, host[l][0], host[l][1], l)
        ref = oa.paged_decode_attention(q[l], kp, vp, tables, lens, B, scale)
        assert_close(got[l], ref, f"B={block_size} layer={l}")
        del kp, vp, ref


def _custom(D, G, B, N=6, lens="uniform:1,300", seed=0):
    return WorkloadSpec(key="custom", title="custom", num_layers=1, num_seqs=N,
                        num_q_heads=2 * G, num_kv_heads=2, head_dim=D, block_size=B, seed=seed,
                        lengths=lens)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
@pytest.mark.parametrize("B", [4, 8, 16, 32])
def test_shape_sweep_with_split_partitions(D, G, B):
    spec = _custom(D, G, B, seed=100 + D + 10 * G + B)
    w = make_workload(spec)
    ref = _oracle_attention(w, 0)
    for part in (64, 0):
        outs = gpu_step(pkv, w, device_inputs(w), partition_tokens=part)
        _assert_no_device_error()
        assert_close(f64(outs[0]), ref, f"D={D} G={G} B={B} part={part}")


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_many_pieces_two_level_merge(D, G):
    # one tile per range: a 4096-token sequence is 128 (d 64) or 256 (d 128)
    # pieces per (sequence, kv head), merged in groups of ranges and then groups;
    # at d 64 a merge fetches 8 / G pieces per round trip (G = 8: one)
    spec = WorkloadSpec(key="custom", title="custom", num_layers=1, num_seqs=3, num_q_heads=2 * G,
                        num_kv_heads=2, head_dim=D, block_size=16, seed=7 + D + G,
                        lengths="fixed:4096,1000,37")
    w = make_workload(spec)
    ref = _oracle_attention(w, 0)
    tile = 32 if D == 64 else 16
    outs = gpu_step(pkv, w, device_inputs(w), partition_tokens=tile)
    _assert_no_device_error()
    assert_close(f64(outs[0]), ref, f"D={D} G={G} one tile per range")
    again = gpu_step(pkv, w, device_inputs(w), partition_tokens=tile)[0]
    assert torch.equal(outs[0].view(torch.int16), again.view(torch.int16))


def test_physical_permutation_invariance():
    """Relabelling physical blocks changes nothing: both runs match the oracle
    and are bit-identical (the work split depends only on the lengths, and
    split pieces are merged in a fixed order)."""
    w = make_workload("continuous_batch")
    out1 = gpu_step(pkv, w, device_inputs(w))[0]
    perm = np.random.default_rng(3).permutation(w.num_blocks)
    w2 = dataclasses.replace(w)
    w2.k_pool = torch.empty_like(w.k_pool)
    w2.v_pool = torch.empty_like(w.v_pool)
    p = torch.from_numpy(perm)
    w2.k_pool[:, p] = w.k_pool
    w2.v_pool[:, p] = w.v_pool
    bt = w.block_tables.copy()
    bt[bt >= 0] = perm[bt[bt >= 0]]
    w2.block_tables = bt
    pairs = perm[w.copy_pairs].astype(np.int32)
    w2.copy_pairs = pairs
    blk, off = np.divmod(w.slot_mapping, w.block_size)
    w2.slot_mapping = perm[blk] * w.block_size + off
    out2 = gpu_step(pkv, w2, device_inputs(w2))[0]
    ref = _oracle_attention(w, 0)
    assert_close(f64(out1), ref, "original ids")
    assert_close(f64(out2), ref, "permuted ids")
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))


def test_workspace_reuse_is_stable():
    w = make_workload("long_context")
    dev = device_inputs(w)
    spec = w.spec
    ws = pkv.make_workspace(w.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim,
                            w.max_blocks, w.block_size, 512)
    a = gpu_step(pkv, w, dev, workspace=ws)[0].clone()
    ref = _oracle_attention(w, 0)
    assert_close(f64(a), ref, "first call")
    for _ in range(3):
        b = gpu_step(pkv, w, dev, workspace=ws)[0]
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # the tickets are back at zero: the workspace ends with the group tickets
    # (units here have 74 pieces, so both merge levels ran), and the later
    # calls above agree bit for bit with the first
    assert int(ws[-256:].view(torch.int32).abs().sum()) == 0
    _assert_no_device_error()


# ---------------------------------------------------------------------------
# edge cases
# ---------------------------------------------------------------------------

def _tiny_problem(lens, B=16, D=64, Hkv=2, G=4, NB=64, seed=5):
    g = torch.Generator().manual_seed(seed)
    kp = torch.randn((NB, Hkv, B, D), generator=g).to(torch.bfloat16)
    vp = torch.randn((NB, Hkv, B, D), generator=g).to(torch.bfloat16)
    q = torch.randn((len(lens), Hkv * G, D), generator=g).to(torch.bfloat16)
    maxb = max(1, max(-(-n // B) for n in lens))
    perm = np.random.default_rng(seed).permutation(NB)
    bt = np.full((len(lens), maxb), -1, np.int32)
    c = 0
    for i, n in enumerate(lens):
        k = -(-n // B)
        bt[i, :k] = perm[c:c + k]
        c += k
    return kp, vp, q, bt


def _run(kp, vp, q, bt, lens, B, scale=0.125, part=0):
    out = torch.full(q.shape, float("nan"), dtype=torch.bfloat16, device="cuda")
    Hkv, D = kp.shape[1], kp.shape[3]
    ws = pkv.make_workspace(q.shape[0], q.shape[1], Hkv, D, bt.shape[1], B, part)
    pkv.paged_decode_attention(q.cuda(), kp.cuda(), vp.cuda(), torch.from_numpy(bt).cuda(),
                               torch.tensor(lens, dtype=torch.int32).cuda(), B, scale, out,
                               workspace=ws, partition_tokens=part)
    torch.cuda.synchronize()
    return out


def test_edge_lengths_zero_one_and_block_multiples():
    B = 16
    lens = [0, 1, 16, 17, 32, 255, 256, 257]
    kp, vp, q, bt = _tiny_problem(lens, B=B)
    for part in (0, 32):
        out = _run(kp, vp, q, bt, lens, B, part=part)
        _assert_no_device_error()
        ref = oa.paged_decode_attention(u16(q), u16(kp), u16(vp), bt, lens, B, 0.125)
        got = f64(out)
        assert np.array_equal(got[0], np.zeros_like(got[0]))          # empty: zeros
        v0 = ob.to_f64(u16(vp)[bt[1, 0], :, 0])                       # one token: its value, exactly
        assert np.array_equal(got[1], np.repeat(v0, 4, axis=0))
        assert_close(got, ref, f"edge part={part}")


def test_empty_batch_is_a_no_op():
    kp, vp, q, bt = _tiny_problem([5])
    out = torch.zeros((0, 8, 64), dtype=torch.bfloat16, device="cuda")
    pkv.paged_decode_attention(q[:0].cuda(), kp.cuda(), vp.cuda(), torch.from_numpy(bt[:0]).cuda(),
                               torch.zeros(0, dtype=torch.int32, device="cuda"), 16, 0.125, out)
    torch.cuda.synchronize()
    _assert_no_device_error()


def test_bad_block_id_and_overlong_sequence_are_reported():
    B = 16
    lens = [40, 20]
    kp, vp, q, bt = _tiny_problem(lens, B=B)
    bad = bt.copy()
    bad[0, 1] = kp.shape[0] + 7            # outside the pool: not fetched, flagged
    _run(kp, vp, q, bad, lens, B)
    assert pkv.get_device_status(reset=True) & pkv.DEV_RANGE
    _run(kp, vp, q, bt, [bt.shape[1] * B + 9, 20], B)   # longer than its table: clamped, flagged
    assert pkv.get_device_status(reset=True) & pkv.DEV_LENGTH
    out = _run(kp, vp, q, bt, lens, B)                   # the context is still usable
    _assert_no_device_error()
    ref = oa.paged_decode_attention(u16(q), u16(kp), u16(vp), bt, lens, B, 0.125)
    assert_close(f64(out), ref, "after faults")


def test_scores_far_from_zero_stay_finite():
    B = 16
    lens = [300, 5]
    kp, vp, q, bt = _tiny_problem(lens, B=B)
    qb = (q.float() * 60).to(torch.bfloat16)
    out = _run(kp, vp, qb, bt, lens, B, scale=1.0, part=64)
    _assert_no_device_error()
    ref = oa.paged_decode_attention(u16(qb), u16(kp), u16(vp), bt, lens, B, 1.0)
    assert_close(f64(out), ref, "large scores")

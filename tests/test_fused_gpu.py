"""GPU parity of the fused decode step (append of each sequence's newest token
and attention in one launch) against the oracle and against the two-call path.

Bars: pools bit exact against the oracle's kv_append (the new slots start
NaN-poisoned, so a missed store shows); attention within
|gpu - oracle| <= 1e-2 + 1e-2 |oracle|, and bit-identical to kv_append
followed by paged_decode_attention (same tiles, same order of arithmetic).
"""

import numpy as np
import pytest
import torch

from oracle import attention as oa
from workload import make_workload
from workload.configs import WorkloadSpec

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


def _fused_vs_oracle_and_two_call(w, partition=None, layers=None, cow=False):
    dev_f = device_inputs(w)
    dev_t = device_inputs(w)
    outs_f = gpu_step(pkv, w, dev_f, layers=layers, partition_tokens=partition, fused=True,
                      cow=cow)
    outs_t = gpu_step(pkv, w, dev_t, layers=layers, partition_tokens=partition)
    assert pkv.get_device_status(reset=True) == 0
    for l, out in outs_f.items():
        # pools: the fused store equals kv_append's, bit for bit
        kp, vp = oracle_pools_after_step(w, u16(w.k_pool[l]), u16(w.v_pool[l]), l)
        assert np.array_equal(u16(dev_f["k_pool"][l]), kp), f"layer {l}: K pool"
        assert np.array_equal(u16(dev_f["v_pool"][l]), vp), f"layer {l}: V pool"
        ref = oa.paged_decode_attention(u16(w.q[l]), kp, vp, w.block_tables, w.seq_lens,
                                        w.block_size, w.spec.scale)
        assert_close(f64(out), ref, f"{w.spec.key} layer {l}")
        assert torch.equal(out.view(torch.int16), outs_t[l].view(torch.int16)), f"layer {l}"


@pytest.mark.parametrize("key", ["tiny", "llama1b_layer", "continuous_batch"])
def test_fused_step_matches_oracle(key):
    _fused_vs_oracle_and_two_call(make_workload(key))


@pytest.mark.parametrize("partition", [0, 64])
def test_fused_copy_on_write_continuous_batch(partition):
    # 28 copy-on-write pairs folded into the attention launch: the copied tails
    # (every head, K and V, NaN-poisoned destinations) must come out bit exact
    w = make_workload("continuous_batch")
    assert len(w.copy_pairs) > 0
    _fused_vs_oracle_and_two_call(w, partition=partition, cow=True)


@pytest.mark.parametrize("D,G,B", [(64, 4, 16), (128, 4, 16), (64, 8, 4), (128, 1, 32), (64, 2, 8)])
def test_fused_copy_on_write_shapes(D, G, B):
    spec = WorkloadSpec(key="custom", title="custom", num_layers=2, num_seqs=20,
                        num_q_heads=2 * G, num_kv_heads=2, head_dim=D, block_size=B,
                        seed=500 + D + G + B, lengths="uniform:1,200", shared_groups=2,
                        shared_group_size=4, shared_prefix=3 * B)
    w = make_workload(spec)
    assert len(w.copy_pairs) > 0
    _fused_vs_oracle_and_two_call(w, partition=0, cow=True)


@pytest.mark.parametrize("partition", [512, 0])
def test_fused_long_context(partition):
    _fused_vs_oracle_and_two_call(make_workload("long_context"), partition=partition)


def _custom(D, G, B, N=6, lens="uniform:1,300", seed=0):
    return WorkloadSpec(key="custom", title="custom", num_layers=2, num_seqs=N,
                        num_q_heads=2 * G, num_kv_heads=2, head_dim=D, block_size=B, seed=seed,
                        lengths=lens)


@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 4, 8])
@pytest.mark.parametrize("B", [4, 16, 32])
def test_fused_shape_sweep(D, G, B):
    w = make_workload(_custom(D, G, B, seed=300 + D + 10 * G + B))
    _fused_vs_oracle_and_two_call(w, partition=64)


def test_fused_lengths_one_and_block_boundaries():
    # length 1: the only token is the new one, so the output is v_new exactly
    # (after the bf16 round trip); lengths at and just past block multiples
    w = make_workload(_custom(64, 4, 16, N=7, lens="fixed:1,16,17,32,33,1,48", seed=9))
    _fused_vs_oracle_and_two_call(w, partition=0)
    dev = device_inputs(w)
    out = gpu_step(pkv, w, dev, fused=True)[0]
    G = w.spec.num_q_heads // w.spec.num_kv_heads
    for s in np.nonzero(w.seq_lens == 1)[0]:
        want = w.v_new[0, s].repeat_interleave(G, dim=0)
        assert torch.equal(out[s].cpu().view(torch.int16), want.view(torch.int16))


def test_fused_binding_checks_new_row_shapes():
    w = make_workload("tiny")
    dev = device_inputs(w)
    out = torch.empty_like(dev["q"][0])
    with pytest.raises(ValueError):
        pkv.append_paged_decode_attention(dev["k_new"][0][:-1], dev["v_new"][0], dev["q"][0],
                                          dev["k_pool"], dev["v_pool"], dev["tables"], dev["lens"],
                                          w.block_size, w.spec.scale, out)


@pytest.mark.parametrize("seed", range(8))
def test_random_shapes_fuzz(seed):
    # random head_dim, group, block size, batch, length mix, sharing and
    # partition cap; the one-launch step (copy-on-write, append, attention)
    # against the oracle and against the two-call path
    rng = np.random.default_rng(1000 + seed)
    D = int(rng.choice([64, 128]))
    G = int(rng.choice([1, 2, 4, 8]))
    B = int(rng.choice([4, 8, 16, 32]))
    Hkv = int(rng.choice([1, 2, 4]))
    N = int(rng.integers(9, 40))
    hi = int(rng.choice([40, 300, 1500]))
    groups = int(rng.integers(0, 3))
    spec = WorkloadSpec(key="custom", title="custom", num_layers=int(rng.integers(1, 3)),
                        num_seqs=N, num_q_heads=Hkv * G, num_kv_heads=Hkv, head_dim=D,
                        block_size=B, seed=2000 + seed, lengths=f"uniform:1,{hi}",
                        shared_groups=groups, shared_group_size=4 if groups else 0,
                        shared_prefix=2 * B if groups else 0)
    w = make_workload(spec)
    part = int(rng.choice([0, 0, 32, 64, 256]))
    _fused_vs_oracle_and_two_call(w, partition=part, cow=bool(groups))


@pytest.mark.parametrize("N", [800, 2500])
def test_batches_past_the_shared_memory_prefix(N):
    # more than 768 sequences: the tile prefix lives in the workspace and the
    # lengths are read from global memory; with copy-on-write groups
    spec = WorkloadSpec(key="custom", title="custom", num_layers=1, num_seqs=N, num_q_heads=4,
                        num_kv_heads=1, head_dim=64, block_size=16, seed=3000 + N,
                        lengths="uniform:1,70", shared_groups=3, shared_group_size=5,
                        shared_prefix=32)
    w = make_workload(spec)
    _fused_vs_oracle_and_two_call(w, partition=0, cow=True)

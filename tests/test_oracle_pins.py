"""Pins for the CPU oracle: values the pages print, closed forms, library
routines and brute force, chosen so that a plausible slip anywhere in the
oracle (dropped scale, wrong sign, wrong index, transposed operand, wrong GQA
mapping, missing max rescale) fails at least one of them.

No GPU is needed; nothing here touches the CUDA path.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch
import torch.nn.functional as F

from oracle import attention as oa
from oracle import bf16 as ob
from oracle import paging as op


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _rand_bf16(rng, shape, scale=1.0):
    """Random values rounded to bf16 bit patterns (test-local, truncating the fp32 draw)."""
    x = (rng.standard_normal(shape) * scale).astype(np.float32)
    return (x.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


# ---------------------------------------------------------------------------
# bf16 widening
# ---------------------------------------------------------------------------

def test_bf16_widening_exact_values():
    bits = np.array([0x3F80, 0xBF80, 0x4000, 0x3E00, 0x0000, 0x8000, 0x7F80, 0x0001], np.uint16)
    want = [1.0, -1.0, 2.0, 0.125, 0.0, -0.0, np.inf, 2.0 ** -133]
    got = ob.to_f64(bits)
    for g, w in zip(got, want):
        assert g == w and math.copysign(1, g) == math.copysign(1, w)
    assert np.isnan(ob.to_f64(np.array([0x7FC0], np.uint16)))[0]
    assert np.array_equal(ob.from_f64_exact([1.0, -2.0, 0.125]), [0x3F80, 0xC000, 0x3E00])
    with pytest.raises(ValueError):
        ob.from_f64_exact([1.0 + 2 ** -10])


def test_bf16_widening_matches_torch():
    rng = np.random.default_rng(0)
    bits = rng.integers(0, 0x7F80, size=4096).astype(np.uint16)
    t = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(ob.to_f64(bits), t)


# ---------------------------------------------------------------------------
# block arithmetic and the block manager
# ---------------------------------------------------------------------------

def test_block_table_growth_worked_example(golden_dir):
    g = _load(golden_dir, "block_table_growth.json")
    B = g["block_size"]
    order = g["free_order_head"] + [b for b in range(8) if b not in g["free_order_head"]]
    bm = op.BlockManager(num_blocks=8, block_size=B, free_order=order)
    assert bm.add_sequence("req", g["prompt_tokens"]) == g["table_after_prompt"]
    for key in ("append_1", "append_2"):
        a = g[key]
        free_before = bm.num_free()
        slot = bm.append_slot("req")
        assert slot == a["physical_block"] * B + a["offset"]
        assert bm.tables["req"] == a["table_after"]
        assert op.translate(bm.tables["req"], a["position"], B) == (a["physical_block"], a["offset"])
        # the first append allocates nothing, the second takes exactly one block
        assert free_before - bm.num_free() == (0 if key == "append_1" else 1)
    assert bm.take_copy_pairs() == []
    bm.free_sequence("req")
    assert sorted(list(bm.free)[-3:]) == sorted(g["released_blocks_return_to_pool"])
    assert bm.num_free() == 8


def test_address_translation_worked_example(golden_dir):
    g = _load(golden_dir, "address_translation.json")
    B, table = g["block_size"], g["block_table"]
    for lk in g["lookups"]:
        assert lk["position"] // B == lk["logical_block"]
        assert op.translate(table, lk["position"], B) == (lk["physical_block"], lk["offset"])
        assert op.flat_slot(table, lk["position"], B) == lk["physical_block"] * B + lk["offset"]
    T = g["num_tokens"]
    assert op.blocks_needed(T, B) == g["blocks_needed"]
    assert op.slots_occupied(T, B) == g["slots_occupied"]
    assert op.slots_occupied(T, B) - T == g["empty_slots"]
    with pytest.raises(IndexError):
        op.translate(table, 12, B)


def test_blocks_needed_brute_force():
    for B in range(1, 34):
        for T in range(0, 200):
            n = op.blocks_needed(T, B)
            # smallest n with n*B >= T
            assert n * B >= T and (n == 0 or (n - 1) * B < T)
            assert 0 <= op.slots_occupied(T, B) - T < B
            assert n == math.ceil(T / B)


def test_translation_is_a_bijection_onto_the_tables_slots():
    """Brute force: every position of a random table lands in a distinct slot of its own blocks."""
    rng = np.random.default_rng(1)
    for B in (1, 4, 8, 16, 32):
        NB = 40
        T = int(rng.integers(1, 8 * B))
        table = rng.permutation(NB)[: op.blocks_needed(T, B)].tolist()
        slots = [op.flat_slot(table, p, B) for p in range(T)]
        assert len(set(slots)) == T
        for p, s in enumerate(slots):
            assert s // B == table[p // B] and s % B == p % B


def test_copy_on_write_worked_example(golden_dir):
    g = _load(golden_dir, "copy_on_write.json")
    B = g["block_size"]
    order = g["free_order_head"] + [b for b in range(8) if b not in g["free_order_head"]]
    bm = op.BlockManager(num_blocks=8, block_size=B, free_order=order)
    assert bm.add_sequence("A", g["shared_tokens"]) == g["table_before"]
    assert bm.fork("A", "B") == g["table_before"]
    assert bm.refcount[3] == 2 and bm.refcount[0] == 2
    slot_a = bm.append_slot("A")
    slot_b = bm.append_slot("B")
    assert bm.take_copy_pairs() == [tuple(p) for p in g["copy_pairs"]]
    assert bm.tables["A"] == g["table_A_after"]
    assert bm.tables["B"] == g["table_B_after"]
    assert divmod(slot_a, B) == tuple(g["slot_A_block_offset"])
    assert divmod(slot_b, B) == tuple(g["slot_B_block_offset"])
    for blk, rc in g["refcount_after"].items():
        assert bm.refcount[int(blk)] == rc

    # the data movement of the same step: copy the tail, then append a and b
    L, H, d = 2, 2, 4
    rng = np.random.default_rng(7)
    kp = _rand_bf16(rng, (L, 8, H, B, d))
    vp = _rand_bf16(rng, (L, 8, H, B, d))
    k2, v2 = oa.block_copy(kp, vp, g["copy_pairs"])
    for layer in range(L):
        ka = _rand_bf16(rng, (2, H, d))
        va = _rand_bf16(rng, (2, H, d))
        k3, v3 = oa.kv_append(k2[layer], v2[layer], ka, va, [slot_a, slot_b], B)
        # the shared full block is never written
        assert np.array_equal(k3[3], kp[layer, 3]) and np.array_equal(v3[3], vp[layer, 3])
        # P4 = the old tail's positions 4-5, then A's token at offset 2
        assert np.array_equal(k3[4, :, :2], kp[layer, 0, :, :2])
        assert np.array_equal(k3[4, :, 2], ka[0]) and np.array_equal(v3[4, :, 2], va[0])
        # P0 keeps positions 4-5 and receives B's token at offset 2
        assert np.array_equal(k3[0, :, :2], kp[layer, 0, :, :2])
        assert np.array_equal(k3[0, :, 2], ka[1]) and np.array_equal(v3[0, :, 2], va[1])


def test_copy_on_write_many_sharers():
    """k sharers of a partial tail: k-1 copies, the last writer keeps the original."""
    B = 16
    bm = op.BlockManager(num_blocks=64, block_size=B)
    bm.add_sequence(0, 512 + 5)
    for c in range(1, 8):
        bm.fork(0, c)
    tail = bm.tables[0][-1]
    full = bm.tables[0][:-1]
    slots = [bm.append_slot(c) for c in range(8)]
    pairs = bm.take_copy_pairs()
    assert len(pairs) == 7 and all(src == tail for src, _ in pairs)
    assert bm.tables[7][-1] == tail and bm.refcount[tail] == 1
    for c in range(8):
        assert bm.tables[c][:-1] == full
        assert slots[c] % B == 5
    assert all(bm.refcount[b] == 8 for b in full)
    # a full shared tail needs no copy: the next token opens a new block
    bm2 = op.BlockManager(num_blocks=16, block_size=4)
    bm2.add_sequence("a", 8)
    bm2.fork("a", "b")
    bm2.append_slot("a")
    bm2.append_slot("b")
    assert bm2.take_copy_pairs() == []


def test_release_returns_shared_blocks_only_with_their_last_user():
    # [PU] 按 Block 分配 / 共享前缀: a finished request drops its references; a
    # block still referenced by another sequence stays out of the pool.  A and
    # B share [P3, P0]; after A's write copied P0 -> P4, A ends: only P4 returns.
    bm = op.BlockManager(8, 4, free_order=[3, 0, 4, 1, 2, 5, 6, 7])
    bm.add_sequence("A", 6)
    bm.fork("A", "B")
    bm.append_slot("A")
    assert bm.tables["A"] == [3, 4] and bm.tables["B"] == [3, 0]
    free_before = list(bm.free)
    bm.free_sequence("A")
    assert list(bm.free) == free_before + [4]
    assert bm.refcount[3] == 1 and bm.refcount[0] == 1
    bm.free_sequence("B")
    assert list(bm.free) == free_before + [4, 3, 0]
    assert all(c == 0 for c in bm.refcount)


def test_block_manager_exhaustion_and_release():
    bm = op.BlockManager(num_blocks=3, block_size=2)
    bm.add_sequence("x", 6)
    with pytest.raises(op.OutOfBlocks):
        bm.append_slot("x")
    bm.free_sequence("x")
    assert bm.num_free() == 3


# ---------------------------------------------------------------------------
# kv_append / block_copy brute force
# ---------------------------------------------------------------------------

def test_kv_append_changes_exactly_the_addressed_slots():
    rng = np.random.default_rng(3)
    NB, H, B, d = 6, 3, 4, 8
    kp = _rand_bf16(rng, (NB, H, B, d))
    vp = _rand_bf16(rng, (NB, H, B, d))
    slots = [5, -1, 22, 0]
    kn = _rand_bf16(rng, (4, H, d))
    vn = _rand_bf16(rng, (4, H, d))
    k2, v2 = oa.kv_append(kp, vp, kn, vn, slots, B)
    changed = np.argwhere(np.any(k2 != kp, axis=(1, 3)) | np.any(v2 != vp, axis=(1, 3)))
    expect = {(s // B, s % B) for s in slots if s >= 0}
    assert {(int(b), int(o)) for b, o in changed} <= expect
    for t, s in enumerate(slots):
        if s < 0:
            continue
        assert np.array_equal(k2[s // B, :, s % B], kn[t])
        assert np.array_equal(v2[s // B, :, s % B], vn[t])
    # NaN payloads and -0 survive (bit patterns are moved, not values)
    odd = np.full((1, H, d), 0x7FC1, np.uint16)
    odd[0, 0, 0] = 0x8000
    k3, _ = oa.kv_append(kp, vp, odd, odd, [9], B)
    assert np.array_equal(k3[2, :, 1], odd[0])
    with pytest.raises(IndexError):
        oa.kv_append(kp, vp, kn[:1], vn[:1], [NB * B], B)


def test_block_copy_all_layers_only_pairs():
    rng = np.random.default_rng(4)
    L, NB, H, B, d = 3, 10, 2, 4, 8
    kp = _rand_bf16(rng, (L, NB, H, B, d))
    vp = _rand_bf16(rng, (L, NB, H, B, d))
    pairs = [(1, 7), (4, 2)]
    k2, v2 = oa.block_copy(kp, vp, pairs)
    for blk in range(NB):
        src = dict((dst, s) for s, dst in pairs).get(blk, blk)
        assert np.array_equal(k2[:, blk], kp[:, src])
        assert np.array_equal(v2[:, blk], vp[:, src])
    k3, v3 = oa.block_copy(kp, vp, np.zeros((0, 2), np.int32))
    assert np.array_equal(k3, kp) and np.array_equal(v3, vp)


def test_swap_out_and_back_in_restores_every_byte():
    # [AKIRA] 故事沒有說完的部分: blocks swapped out to host memory and brought back
    # later.  Round trip through a host pool into other free device blocks gives
    # the original bytes; the source pool is untouched; within one pool a swap is
    # the (separately pinned) block copy.
    rng = np.random.default_rng(12)
    L, NB, NH, H, B, d = 2, 12, 6, 2, 4, 8
    dk = _rand_bf16(rng, (L, NB, H, B, d))
    dv = _rand_bf16(rng, (L, NB, H, B, d))
    hk = np.zeros((L, NH, H, B, d), np.uint16)
    hv = np.zeros((L, NH, H, B, d), np.uint16)
    out = [(3, 0), (7, 5), (0, 2)]
    hk2, hv2 = oa.swap_blocks(dk, dv, hk, hv, out)
    for s, t in out:
        assert np.array_equal(hk2[:, t], dk[:, s]) and np.array_equal(hv2[:, t], dv[:, s])
    assert not hk2[:, [1, 3, 4]].any() and not hv2[:, [1, 3, 4]].any()
    back = [(0, 9), (5, 10), (2, 11)]
    dk2, dv2 = oa.swap_blocks(hk2, hv2, dk, dv, back)
    for (s, _), (_, t) in zip(out, back):
        assert np.array_equal(dk2[:, t], dk[:, s]) and np.array_equal(dv2[:, t], dv[:, s])
    keep = [b for b in range(NB) if b not in (9, 10, 11)]
    assert np.array_equal(dk2[:, keep], dk[:, keep]) and np.array_equal(dv2[:, keep], dv[:, keep])
    same = oa.swap_blocks(dk, dv, dk, dv, [(1, 7), (4, 2)])
    ref = oa.block_copy(dk, dv, [(1, 7), (4, 2)])
    assert np.array_equal(same[0], ref[0]) and np.array_equal(same[1], ref[1])


# ---------------------------------------------------------------------------
# the merge rule
# ---------------------------------------------------------------------------

def test_merge_worked_example(golden_dir):
    g = _load(golden_dir, "partition_merge.json")
    rng = np.random.default_rng(5)
    o1, o2 = rng.standard_normal(16), rng.standard_normal(16)
    # equal max scores: the Z's are the page's Z's
    _, Z, o = oa.merge([(0.0, g["Z"][0], o1), (0.0, g["Z"][1], o2)])
    assert Z == sum(g["Z"])
    np.testing.assert_allclose(o, g["weights"][0] * o1 + g["weights"][1] * o2, rtol=0, atol=1e-15)
    # the same weights when the partials are stored on different max bases
    m1, m2 = 5.0, -2.0
    Z1 = g["Z"][0] * math.exp(-m1)  # Z_r = sum e^{s - m_r}: same e^{s} sums, other bases
    Z2 = g["Z"][1] * math.exp(-m2)
    _, _, o = oa.merge([(m1, Z1, o1), (m2, Z2, o2)])
    np.testing.assert_allclose(o, 0.75 * o1 + 0.25 * o2, rtol=0, atol=1e-14)


def test_merge_is_associative_and_handles_empty():
    rng = np.random.default_rng(6)
    parts = [(rng.standard_normal() * 10, rng.random() + 0.1, rng.standard_normal(8)) for _ in range(5)]
    flat = oa.merge(parts)
    step = parts[0]
    for p in parts[1:]:
        step = oa.merge([step, p])
    tree = oa.merge([oa.merge(parts[:2]), oa.merge(parts[2:])])
    np.testing.assert_allclose(step[2], flat[2], atol=1e-13)
    np.testing.assert_allclose(tree[2], flat[2], atol=1e-13)
    empty = (-np.inf, 0.0, np.zeros(8))
    np.testing.assert_array_equal(oa.merge(parts + [empty])[2], flat[2])
    assert oa.merge([empty])[1] == 0.0


def test_merge_survives_scores_that_overflow_exp():
    """Max rescale: scores near 1000 overflow e^{s} in fp64 but merge fine."""
    v1, v2 = np.array([1.0, 0.0]), np.array([0.0, 1.0])
    parts = [oa.partial(np.array([1.0]), np.array([[1000.0]]), v1[None], 1.0),
             oa.partial(np.array([1.0]), np.array([[1000.0 - math.log(3.0)]]), v2[None], 1.0)]
    assert np.isinf(np.exp(1000.0))
    o = oa.merge(parts)[2]
    np.testing.assert_allclose(o, [0.75, 0.25], atol=1e-12)


# ---------------------------------------------------------------------------
# attention: closed forms, a library routine, invariances
# ---------------------------------------------------------------------------

def _identity_case(rng, N, Hq, Hkv, d, B, lens):
    maxb = max(op.blocks_needed(n, B) for n in lens)
    NB = N * maxb
    tables = np.arange(NB, dtype=np.int32).reshape(N, maxb)
    q = _rand_bf16(rng, (N, Hq, d))
    kp = _rand_bf16(rng, (NB, Hkv, B, d))
    vp = _rand_bf16(rng, (NB, Hkv, B, d))
    return q, kp, vp, tables


def test_two_token_closed_form():
    """Scores scale*q.k = ln 3 and 0 give weights 3/4, 1/4 (the page's example)."""
    d, B = 4, 4
    q = ob.from_f64_exact([[[1.0, 0.0, 0.0, 0.0]]])
    kp = np.zeros((1, 1, B, d), np.uint16)
    vp = np.zeros((1, 1, B, d), np.uint16)
    kp[0, 0, 0] = ob.from_f64_exact([1.0, 0.0, 0.0, 0.0])   # s = scale
    kp[0, 0, 1] = ob.from_f64_exact([0.0, 0.0, 0.0, 0.0])   # s = 0
    vp[0, 0, 0] = ob.from_f64_exact([1.0, 2.0, 0.0, -4.0])
    vp[0, 0, 1] = ob.from_f64_exact([0.0, -2.0, 8.0, 4.0])
    kp[0, 0, 2:] = ob.BF16_QNAN   # unused slots must never be read
    vp[0, 0, 2:] = ob.BF16_QNAN
    out = oa.paged_decode_attention(q, kp, vp, [[0]], [2], B, math.log(3.0))
    np.testing.assert_allclose(out[0, 0], [0.75, 1.0, 2.0, -2.0], atol=1e-14)
    # 1/sqrt(d) as the scale: s1 = 1/2 -> weight e^{0.5}/(e^{0.5}+1)
    out = oa.paged_decode_attention(q, kp, vp, [[0]], [2], B, 1.0 / math.sqrt(d))
    w = math.exp(0.5) / (math.exp(0.5) + 1.0)
    np.testing.assert_allclose(out[0, 0], w * np.array([1, 2, 0, -4]) + (1 - w) * np.array([0, -2, 8, 4]),
                               atol=1e-14)


def test_identity_table_equals_library_dense_attention():
    """Identity block table == torch SDPA (fp64, GQA) on contiguous K/V."""
    rng = np.random.default_rng(8)
    N, Hq, Hkv, d, B = 3, 8, 2, 16, 4
    lens = [5, 12, 1]
    q, kp, vp, tables = _identity_case(rng, N, Hq, Hkv, d, B, lens)
    out = oa.paged_decode_attention(q, kp, vp, tables, lens, B, 1 / math.sqrt(d))
    maxb = tables.shape[1]
    for s, n in enumerate(lens):
        # contiguous [Hkv, maxb*B, d] view of this sequence's blocks
        Kc = ob.to_f64(kp[tables[s]]).transpose(1, 0, 2, 3).reshape(Hkv, maxb * B, d)[:, :n]
        Vc = ob.to_f64(vp[tables[s]]).transpose(1, 0, 2, 3).reshape(Hkv, maxb * B, d)[:, :n]
        qs = torch.from_numpy(ob.to_f64(q[s]))[None, :, None, :]
        ref = F.scaled_dot_product_attention(qs, torch.from_numpy(Kc)[None], torch.from_numpy(Vc)[None],
                                             scale=1 / math.sqrt(d), enable_gqa=True)
        np.testing.assert_allclose(out[s], ref[0, :, 0].numpy(), rtol=0, atol=1e-12)
        # and scipy's softmax, head by head
        G = Hq // Hkv
        for h in range(Hq):
            p = scipy.special.softmax(Kc[h // G] @ ob.to_f64(q[s, h]) / math.sqrt(d))
            np.testing.assert_allclose(out[s, h], p @ Vc[h // G], rtol=0, atol=1e-12)


def test_gqa_mapping_and_mha_special_case():
    """G = 1 is multi-head attention; with G = 4, heads 0-3 read kv head 0 only."""
    rng = np.random.default_rng(9)
    d, B = 8, 4
    q, kp, vp, tables = _identity_case(rng, 1, 8, 2, d, B, [7])
    out = oa.paged_decode_attention(q, kp, vp, tables, [7], B, 0.3)
    # poison kv head 1: heads 0..3 must not change, heads 4..7 must
    kp2 = kp.copy()
    kp2[:, 1] = ob.from_f64_exact(np.full(d, 2.0))
    out2 = oa.paged_decode_attention(q, kp2, vp, tables, [7], B, 0.3)
    assert np.array_equal(out[0, :4], out2[0, :4])
    assert not np.allclose(out[0, 4:], out2[0, 4:])
    # MHA: each head against its own kv head equals a 1-head problem
    q1, kp1, vp1, t1 = _identity_case(rng, 1, 2, 2, d, B, [6])
    full = oa.paged_decode_attention(q1, kp1, vp1, t1, [6], B, 0.5)
    for h in range(2):
        one = oa.paged_decode_attention(q1[:, h:h + 1], kp1[:, h:h + 1], vp1[:, h:h + 1], t1, [6], B, 0.5)
        assert np.array_equal(one[0, 0], full[0, h])


def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(10)
    q, kp, vp, tables = _identity_case(rng, 1, 4, 1, 16, 8, [1])
    out = oa.paged_decode_attention(q, kp, vp, tables, [1], 8, 0.25)
    for h in range(4):
        assert np.array_equal(out[0, h], ob.to_f64(vp[tables[0, 0], 0, 0]))


def test_equal_keys_give_the_mean_of_values():
    rng = np.random.default_rng(11)
    d, B, n = 8, 4, 11
    q, kp, vp, tables = _identity_case(rng, 1, 2, 1, d, B, [n])
    kp[:] = kp[0, 0, 0]
    out = oa.paged_decode_attention(q, kp, vp, tables, [n], B, 0.7)
    Vc = ob.to_f64(vp[tables[0]]).reshape(-1, d)[:n]
    np.testing.assert_allclose(out[0, 0], Vc.mean(axis=0), atol=1e-14)


def test_huge_scores_do_not_overflow_and_pick_the_argmax():
    rng = np.random.default_rng(12)
    d, B, n = 16, 4, 9
    q, kp, vp, tables = _identity_case(rng, 1, 1, 1, d, B, [n])
    qf = ob.to_f64(q) * 1000.0
    q_big = (qf.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    out = oa.paged_decode_attention(q_big, kp, vp, tables, [n], B, 1.0)
    assert np.all(np.isfinite(out))
    K = oa.gather_tokens(kp, tables[0], range(n), B, 0)
    V = oa.gather_tokens(vp, tables[0], range(n), B, 0)
    s = K @ ob.to_f64(q_big[0, 0])
    top = np.argsort(s)[-2:]
    if s[top[1]] - s[top[0]] > 50:  # the winner dominates completely
        np.testing.assert_allclose(out[0, 0], V[top[1]], atol=1e-12)
    # no-rescale exp(s) overflows here: the definition must subtract the max
    assert np.isinf(np.exp(s.max()))


def test_physical_block_permutation_invariance():
    rng = np.random.default_rng(13)
    N, Hq, Hkv, d, B = 4, 8, 2, 16, 4
    lens = [7, 9, 1, 16]
    q, kp, vp, tables = _identity_case(rng, N, Hq, Hkv, d, B, lens)
    out = oa.paged_decode_attention(q, kp, vp, tables, lens, B, 0.25)
    perm = rng.permutation(kp.shape[0])          # block b moves to perm[b]
    kp2 = np.empty_like(kp)
    vp2 = np.empty_like(vp)
    kp2[perm] = kp
    vp2[perm] = vp
    out2 = oa.paged_decode_attention(q, kp2, vp2, perm[tables], lens, B, 0.25)
    assert np.array_equal(out, out2)


def test_table_entries_past_the_length_are_never_read():
    rng = np.random.default_rng(14)
    q, kp, vp, tables = _identity_case(rng, 2, 4, 2, 8, 4, [5, 8])
    out = oa.paged_decode_attention(q, kp, vp, tables, [5, 8], 4, 0.5)
    t2 = np.concatenate([tables, np.full((2, 3), -1, np.int32)], axis=1)
    kp2, vp2 = kp.copy(), vp.copy()
    kp2[tables[0, 1], :, 1:] = ob.BF16_QNAN   # slots past position 4 of sequence 0
    vp2[tables[0, 1], :, 1:] = ob.BF16_QNAN
    out2 = oa.paged_decode_attention(q, kp2, vp2, t2, [5, 8], 4, 0.5)
    assert np.array_equal(out, out2)


def test_split_partitions_match_single_pass():
    rng = np.random.default_rng(15)
    N, Hq, Hkv, d, B = 3, 4, 2, 8, 4
    lens = [13, 40, 2]
    q, kp, vp, tables = _identity_case(rng, N, Hq, Hkv, d, B, lens)
    ref = oa.paged_decode_attention(q, kp, vp, tables, lens, B, 0.35)
    for pt in (1, B, 7, 16, 512):
        got = oa.paged_decode_attention_split(q, kp, vp, tables, lens, B, 0.35, pt)
        np.testing.assert_allclose(got, ref, rtol=0, atol=1e-12)


def test_zero_length_sequence_gives_zeros():
    rng = np.random.default_rng(16)
    q, kp, vp, tables = _identity_case(rng, 2, 2, 1, 8, 4, [3, 1])
    out = oa.paged_decode_attention(q, kp, vp, tables, [3, 0], 4, 0.5)
    assert np.array_equal(out[1], np.zeros((2, 8)))
    assert np.all(np.isfinite(out[0]))


def test_attention_rows_matches_full():
    rng = np.random.default_rng(17)
    N, Hq, Hkv, d, B = 3, 8, 2, 8, 4
    lens = [6, 11, 3]
    q, kp, vp, tables = _identity_case(rng, N, Hq, Hkv, d, B, lens)
    full = oa.paged_decode_attention(q, kp, vp, tables, lens, B, 0.4)
    rows = oa.attention_rows(q, kp, vp, tables[1], lens[1], B, 0.4, 1, [0, 5, 7])
    for h, o in rows.items():
        assert np.array_equal(o, full[1, h])

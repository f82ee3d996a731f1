"""Pins of the prefix-cache block hash oracle: FNV-1a against its published
test vectors, and the properties the pages ask of the block hash (whole
prefix must match, full blocks only, context keys separate caches)."""

import json
import os

import numpy as np

from oracle import prefix_hash as ph

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_fnv1a64_published_vectors():
    with open(os.path.join(GOLDEN, "fnv1a64_vectors.json")) as f:
        rec = json.load(f)
    for v in rec["vectors"]:
        assert ph.fnv1a64(v["input_ascii"].encode()) == int(v["fnv1a64"], 16)


def test_fnv1a64_is_byte_at_a_time():
    # hashing in two pieces, carrying the state, equals hashing the whole
    assert ph.fnv1a64(b"bar", ph.fnv1a64(b"foo")) == ph.fnv1a64(b"foobar")


def test_only_full_blocks_are_hashed():
    toks = list(range(100, 139))
    assert len(ph.prefix_block_hashes(toks, 39, 16)) == 2
    assert len(ph.prefix_block_hashes(toks, 32, 16)) == 2
    assert len(ph.prefix_block_hashes(toks, 15, 16)) == 0


def test_shared_prefix_gives_shared_hashes_and_whole_prefix_must_match():
    rng = np.random.default_rng(0)
    prefix = rng.integers(0, 128256, 48).tolist()
    a = prefix + rng.integers(0, 128256, 16).tolist()
    b = prefix + rng.integers(0, 128256, 16).tolist()
    ha, hb = ph.prefix_block_hashes(a, 64, 16), ph.prefix_block_hashes(b, 64, 16)
    assert ha[:3] == hb[:3] and ha[3] != hb[3]
    # the same block of tokens after a different prefix hashes differently
    c = rng.integers(0, 128256, 16).tolist() + prefix[16:48] + a[48:]
    hc = ph.prefix_block_hashes(c, 64, 16)
    assert hc[1] != ha[1] and hc[2] != ha[2] and hc[3] != ha[3]
    # changing one token changes that block's hash and every later one, none before
    d = list(a)
    d[20] += 1
    hd = ph.prefix_block_hashes(d, 64, 16)
    assert hd[0] == ha[0] and all(x != y for x, y in zip(hd[1:], ha[1:]))


def test_extra_key_separates_caches():
    toks = list(range(64))
    h0 = ph.prefix_block_hashes(toks, 64, 16, extra_key=0)
    h1 = ph.prefix_block_hashes(toks, 64, 16, extra_key=7)
    assert all(x != y for x, y in zip(h0, h1))


def test_chain_definition_on_a_tiny_case():
    # block 0 of [1, 2] with B = 2: digest over 8 token bytes then 8 key bytes,
    # then FNV-1a over 8 zero bytes (no parent) and the digest
    data = (1).to_bytes(4, "little") + (2).to_bytes(4, "little") + bytes(8)
    c = ph.fnv1a64(data)
    assert ph.prefix_block_hashes([1, 2], 2, 2) == [ph.fnv1a64(bytes(8) + c.to_bytes(8, "little"))]

"""The C ABI library builds, loads and exports every symbol include/pagedkv.h
declares; its host-side argument checks answer before any launch (no GPU
needed: every call here returns before touching the device)."""

import ctypes
import os
import re
import subprocess


import paged_kv_cache_378_b200 as pkv
from paged_kv_cache_378_b200 import _lib
from paged_kv_cache_378_b200.build import INCLUDE

HEADER = os.path.join(INCLUDE, "pagedkv.h")


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pkv_[a-z_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert _declared() == sorted(_lib.SIGNATURES)


def test_library_loads_and_exports_every_declared_symbol():
    lib = pkv.library()
    for name in _declared():
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.lib_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (pkv_[a-z_]+)$", out, flags=re.M))
    assert set(_declared()) <= exported


def test_library_is_built_from_these_sources():
    # the loaded library carries the hash of the checkout's sources, header
    # and flags, both in its exported string and in the file the loader scans
    from paged_kv_cache_378_b200 import build as b
    lib = pkv.library()
    assert lib.pkv_build_hash().decode() == b.source_hash()
    assert b.built_hash(_lib.lib_path()) == b.source_hash()
    assert not b.needs_build(_lib.lib_path())


def test_version_and_error_strings():
    lib = pkv.library()
    assert lib.pkv_abi_version() == 1
    for code in range(0, -10, -1):
        assert lib.pkv_strerror(code)
    assert b"unknown" in lib.pkv_strerror(-99)


def _cache(**kw):
    d = dict(k_pool=16, v_pool=32, num_layers=1, num_blocks=8, num_kv_heads=2, block_size=16,
             head_dim=64)
    d.update(kw)
    return _lib.PkvCache(d["k_pool"], d["v_pool"], d["num_layers"], d["num_blocks"],
                         d["num_kv_heads"], d["block_size"], d["head_dim"])


def test_host_argument_checks_before_launch():
    lib = pkv.library()
    P = ctypes.byref
    c = _cache()
    # NULL cache / pools
    assert lib.pkv_kv_append(None, 0, 16, 16, 16, 1, None) == -1
    assert lib.pkv_block_copy(P(_cache(k_pool=0)), 16, 1, None) == -1
    # unsupported shapes
    assert lib.pkv_kv_append(P(_cache(head_dim=96)), 0, 16, 16, 16, 1, None) == -5
    assert lib.pkv_kv_append(P(_cache(block_size=12)), 0, 16, 16, 16, 1, None) == -5
    assert lib.pkv_kv_append(P(_cache(num_blocks=0)), 0, 16, 16, 16, 1, None) == -2
    # misaligned pool / inputs
    assert lib.pkv_kv_append(P(_cache(k_pool=18)), 0, 16, 16, 16, 1, None) == -3
    assert lib.pkv_kv_append(P(c), 0, 24, 16, 16, 1, None) == -3
    # layer range, negative counts, empty work (returns before any launch)
    assert lib.pkv_kv_append(P(c), 1, 16, 16, 16, 1, None) == -7
    assert lib.pkv_kv_append(P(c), 0, 16, 16, 16, -1, None) == -2
    assert lib.pkv_kv_append(P(c), 0, None, None, None, 0, None) == 0
    assert lib.pkv_block_copy(P(c), None, 0, None) == 0
    assert lib.pkv_block_copy(P(c), None, 3, None) == -1
    assert lib.pkv_block_copy(P(c), 16, -2, None) == -2
    att = lib.pkv_paged_decode_attention
    # H_q not a multiple of H_kv, unsupported group, bad scale
    assert att(P(c), 0, 16, 2, 3, 16, 4, 16, 0.125, 16, None, 0, 0, None) == -2
    assert att(P(c), 0, 16, 2, 6, 16, 4, 16, 0.125, 16, None, 0, 0, None) == -5
    assert att(P(c), 0, 16, 2, 8, 16, 4, 16, float("nan"), 16, None, 0, 0, None) == -2
    assert att(P(c), 0, 16, 0, 8, 16, 4, 16, 0.125, 16, None, 0, 0, None) == 0
    assert att(P(c), 0, None, 2, 8, 16, 4, 16, 0.125, 16, None, 0, 0, None) == -1
    assert att(P(c), 0, 16, 2, 8, 16, 4, 16, 0.125, 40, None, 0, 0, None) == -3
    # the workspace is required and must be large enough
    assert att(P(c), 0, 16, 2, 8, 16, 4096, 16, 0.125, 16, None, 0, 512, None) == -4
    need = lib.pkv_attention_workspace_bytes(2, 8, 2, 64, 4096, 16, 512)
    assert need > 0
    assert att(P(c), 0, 16, 2, 8, 16, 4096, 16, 0.125, 16, 256, need - 1, 512, None) == -4
    # fused append + attention: both new-row pointers required and aligned
    fa = lib.pkv_append_paged_decode_attention
    assert fa(P(c), 0, None, 16, None, 16, 2, 8, 16, 4, 16, 0.125, 16, 256, need, 512, None) == -1
    assert fa(P(c), 0, 16, None, None, 16, 2, 8, 16, 4, 16, 0.125, 16, 256, need, 512, None) == -1
    assert fa(P(c), 0, 24, 16, None, 16, 2, 8, 16, 4, 16, 0.125, 16, 256, need, 512, None) == -3
    assert fa(P(c), 0, 16, 16, None, 16, 2, 6, 16, 4, 16, 0.125, 16, 256, need, 512, None) == -5
    assert fa(P(c), 0, 16, 16, None, 16, 0, 8, 16, 4, 16, 0.125, 16, None, 0, 0, None) == 0
    # block copy with a device-side count: the count pointer is required
    assert lib.pkv_block_copy_device_count(P(c), 16, 4, None, None) == -1
    assert lib.pkv_block_copy_device_count(P(c), 16, 0, None, None) == 0
    assert lib.pkv_block_copy_device_count(P(c), 16, -1, 16, None) == -2
    # block swap: the host pool must match the device pool's shape; valid direction
    sw = lib.pkv_swap_blocks
    assert sw(P(c), P(_cache(head_dim=128)), 16, 1, 0, None) == -2
    assert sw(P(c), P(_cache(num_layers=2)), 16, 1, 0, None) == -2
    assert sw(P(c), P(_cache(num_blocks=3)), 16, 1, 2, None) == -2
    assert sw(P(c), P(_cache(num_blocks=3)), 16, 0, 0, None) == 0
    assert sw(P(c), P(_cache(num_blocks=3)), None, 2, 1, None) == -1
    assert sw(P(c), P(_cache(k_pool=0)), 16, 1, 0, None) == -1
    # prefix hashes: resuming (first_block) needs the parent hashes
    ph = lib.pkv_prefix_block_hashes
    assert ph(16, 64, 16, None, 16, None, 4, 16, 16, 4, None) == -1
    assert ph(16, 64, 16, None, None, None, 0, 16, 16, 4, None) == 0
    # device block manager step: state required, sizes checked, at most 4096 sequences
    st = _lib.PkvBlockState(16, 16, 16, 16, 16)
    bm = lib.pkv_block_manager_step
    assert bm(None, 4, 8, 64, 16, None, 16, 16, 16, None, None) == -1
    assert bm(P(st), -1, 8, 64, 16, None, 16, 16, 16, None, None) == -2
    assert bm(P(st), 4, 0, 64, 16, None, 16, 16, 16, None, None) == -2
    assert bm(P(st), 4097, 8, 64, 16, None, 16, 16, 16, None, None) == -5
    assert bm(P(st), 0, 8, 64, 16, None, 16, 16, 16, None, None) == 0
    assert bm(P(st), 4, 8, 64, 16, None, None, 16, 16, None, None) == -1
    assert bm(P(_lib.PkvBlockState(16, 0, 16, 16, 16)), 4, 8, 64, 16, None, 16, 16, 16, None, None) == -1
    # device release: state and rows required, at most num_seqs rows, at most 4096 sequences
    rel = lib.pkv_block_manager_release
    assert rel(None, 4, 8, 64, 16, 16, 2, None) == -1
    assert rel(P(st), 4, 8, 64, 16, 16, 5, None) == -2
    assert rel(P(st), 4, 8, 64, 16, 16, -1, None) == -2
    assert rel(P(st), 4097, 8, 64, 16, 16, 2, None) == -5
    assert rel(P(st), 4, 8, 64, 16, None, 0, None) == 0
    assert rel(P(st), 4, 8, 64, 16, None, 2, None) == -1
    assert rel(P(_lib.PkvBlockState(16, 16, 0, 16, 16)), 4, 8, 64, 16, 16, 2, None) == -1


def test_workspace_and_partition_sizes():
    lib = pkv.library()
    # a requested partition rounds up to the tile: 32 tokens at head_dim 64 (16 with
    # 4-token blocks), 16 at head_dim 128, never less than one block
    assert lib.pkv_partition_tokens(8, 8, 128, 2048, 16, 500) == 512
    assert lib.pkv_partition_tokens(8, 8, 128, 2048, 32, 40) == 64
    assert lib.pkv_partition_tokens(8, 8, 64, 2048, 8, 1) == 32
    assert lib.pkv_partition_tokens(8, 8, 64, 2048, 16, 33) == 64
    assert lib.pkv_partition_tokens(8, 8, 64, 2048, 4, 20) == 32
    assert lib.pkv_partition_tokens(8, 8, 96, 2048, 8, 1) == -1
    assert lib.pkv_partition_tokens(64, 8, 64, 128, 16, 0) == 0      # no cap: even split
    # the workspace holds two partials per range (one range per warp of the grid,
    # more under a cap): (m, Z) + d floats for each of G heads, and a ticket per
    # (sequence, kv head); a cap of C tokens adds ceil(N*Hkv*max_tiles / C) ranges
    n0 = lib.pkv_attention_workspace_bytes(8, 32, 8, 128, 2048, 16, 0)
    n1 = lib.pkv_attention_workspace_bytes(8, 32, 8, 128, 2048, 16, 512)
    units = 8 * 8
    per_range = 2 * 4 * (2 + 128) * 4
    assert n0 >= 148 * 4 * per_range + units * 4
    assert n1 - n0 >= (units * 2048 // 32) * per_range
    # more than 768 sequences: the tile prefix lives in the workspace too
    big = lib.pkv_attention_workspace_bytes(2048, 32, 8, 64, 16, 16, 0)
    small = lib.pkv_attention_workspace_bytes(768, 32, 8, 64, 16, 16, 0)
    assert big - small >= 2049 * 8
    assert lib.pkv_attention_workspace_bytes(8, 30, 8, 128, 2048, 16, 512) == 0
    assert lib.pkv_attention_workspace_bytes(8, 32, 8, 128, 2048, 12, 512) == 0

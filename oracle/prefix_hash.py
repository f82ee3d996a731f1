"""Prefix-cache block hashes (oracle; test infrastructure only).

What the pages fix, restated ("Infra: PagedAttention", section 共享前缀，分叉时
Copy-on-write, the paragraphs on Automatic Prefix Caching): cached blocks are
found again by a hash; only full blocks are cached; a block can be reused only
when the whole prefix before it matches, so its hash covers the hash of the
block before it, the block's own tokens, and context identifiers such as a
LoRA id.

Readings where the pages are silent:

* The hash function is FNV-1a, 64-bit, by its published definition
  (Fowler, Noll, Vo): h = 0xcbf29ce484222325; for each byte b:
  h = (h xor b) * 0x100000001b3 mod 2^64.
* Block b of a sequence: digest c_b = FNV-1a(tokens of the block as int32
  little-endian, then the sequence's extra key as uint64 little-endian);
  hash h_b = FNV-1a(h_{b-1} as uint64 LE, then c_b as uint64 LE), with
  h_{-1} = 0.  So h_b depends on the parent hash, the block's tokens and the
  extra key, as the pages ask, and the per-block digests can be computed
  independently.
* Only blocks b < len // B (full blocks) get a hash.
"""

FNV_OFFSET = 0xCBF29CE484222325
FNV_PRIME = 0x100000001B3
_MASK = (1 << 64) - 1


def fnv1a64(data, h=FNV_OFFSET):
    """FNV-1a 64 over a bytes-like object."""
    for b in bytes(data):
        h ^= b
        h = (h * FNV_PRIME) & _MASK
    return h


def _u64(x):
    return (int(x) & _MASK).to_bytes(8, "little")


def block_digest(block_tokens, extra_key=0):
    """c_b: FNV-1a of the block's tokens (int32 LE) then the extra key (uint64 LE)."""
    data = b"".join((int(t) & 0xFFFFFFFF).to_bytes(4, "little") for t in block_tokens)
    return fnv1a64(data + _u64(extra_key))


def chain(parent, digest):
    """h_b from the parent's hash and the block's digest."""
    return fnv1a64(_u64(parent) + _u64(digest))


def prefix_block_hashes(tokens, length, block_size, extra_key=0):
    """Hashes of the full blocks of one sequence (``tokens`` int, at least ``length`` long)."""
    out = []
    parent = 0
    for b in range(int(length) // block_size):
        h = chain(parent, block_digest(tokens[b * block_size:(b + 1) * block_size], extra_key))
        out.append(h)
        parent = h
    return out

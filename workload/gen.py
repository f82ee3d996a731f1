"""Seeded generator of paged-decode workloads.

Recipe (every draw is seeded; metadata with ``numpy.random.default_rng(seed)``,
values with a ``torch.Generator`` seeded from the same number on the device
the tensors are made on):

1. Lengths.  Each sequence's attention length ``len_s`` counts the token
   appended this step.  ``uniform:a,b`` draws integers in [a, b];
   ``lognormal:median,sigma,lo,hi`` rounds a log-normal draw and clips it;
   ``fixed`` lists them.
2. Physical blocks.  The pool has ``ceil(1.25 x blocks in use)`` blocks
   (or a fixed count); a seeded permutation of all block ids is the free
   list, and sequences take blocks from its front in batch order, so
   physical ids are scattered.
3. Shared prefixes (continuous-batch mix).  Each group of 8 sequences shares
   ``512 + r_g`` cached tokens (``r_g`` seeded in [1, B-1], so the shared
   tail block is partial).  The first 7 writers of a group receive a fresh
   block for the tail and a (shared tail, fresh block) copy pair; the last
   writer keeps the original tail.  All 8 then append one token at offset
   ``r_g``.
4. The new token.  Every sequence appends exactly one token, at position
   ``len_s - 1``; its slot is given in the library's flat slot numbering,
   ``block * B + row``, with the block being the sequence's tail block.
5. Values.  q ``[L, N, H_q, d]``, k_new / v_new ``[L, N, H_kv, d]`` and the
   pools ``[L, NB, H_kv, B, d]`` are N(0, 1) draws rounded to bf16
   (round-to-nearest-even).  With ``poison=True`` every slot that holds no
   live KV before the step (free blocks, copy destinations, tail slots, the
   new token's slot) is set to a bf16 quiet NaN, so any read of a slot the
   step must not read shows up as NaN.
"""

import math
from dataclasses import dataclass
from typing import Optional

import numpy as np
import torch

from .configs import WorkloadSpec, get_spec

BF16_NAN_BITS = 0x7FC0


def rank_seed(seed, rank):
    """Seed of rank ``rank``'s independent batch (rank 0 keeps ``seed``)."""
    return int(seed) + 7919 * int(rank)


def _draw_lengths(recipe, n, rng):
    kind, _, args = recipe.partition(":")
    if kind == "fixed":
        vals = [int(x) for x in args.split(",")]
        if len(vals) != n:
            raise ValueError("fixed length list must have one entry per sequence")
        return np.array(vals, dtype=np.int64)
    if kind == "fixed_all":
        return np.full(n, int(args), dtype=np.int64)
    if kind == "uniform":
        lo, hi = (int(x) for x in args.split(","))
        return rng.integers(lo, hi + 1, size=n).astype(np.int64)
    if kind == "lognormal":
        med, sigma, lo, hi = (float(x) for x in args.split(","))
        x = np.rint(rng.lognormal(math.log(med), sigma, size=n))
        return np.clip(x, lo, hi).astype(np.int64)
    raise ValueError(f"unknown length recipe {recipe!r}")


def _nblocks(n, B):
    return -(-int(n) // B)


@dataclass
class Workload:
    spec: WorkloadSpec
    block_size: int
    num_blocks: int
    seq_lens: np.ndarray          # int32 [N], post-append
    block_tables: np.ndarray      # int32 [N, max_blocks], -1 past each sequence's blocks
    slot_mapping: np.ndarray      # int64 [N]
    copy_pairs: np.ndarray        # int32 [n_pairs, 2] (src, dst)
    live_before: np.ndarray       # bool [NB, B]: slot holds KV before the step
    free_order: Optional[np.ndarray] = None   # the seeded free list, front first
    batch_order: Optional[np.ndarray] = None  # batch position of the i-th sequence drawn
    q: Optional[torch.Tensor] = None        # bf16 [L, N, Hq, d]
    k_new: Optional[torch.Tensor] = None    # bf16 [L, N, Hkv, d]
    v_new: Optional[torch.Tensor] = None
    k_pool: Optional[torch.Tensor] = None   # bf16 [L, NB, Hkv, B, d]
    v_pool: Optional[torch.Tensor] = None
    seed: int = 0

    # -- sizes ------------------------------------------------------------
    @property
    def num_seqs(self):
        return int(self.seq_lens.shape[0])

    @property
    def max_blocks(self):
        return int(self.block_tables.shape[1])

    @property
    def shape(self):
        s = self.spec
        return dict(L=s.num_layers, N=self.num_seqs, Hq=s.num_q_heads, Hkv=s.num_kv_heads,
                    d=s.head_dim, B=self.block_size, NB=self.num_blocks)

    def kv_bytes_read(self):
        """K+V bytes of every valid token of every sequence, one layer."""
        s = self.spec
        return int(self.seq_lens.astype(np.int64).sum()) * 2 * s.num_kv_heads * s.head_dim * 2

    def unique_kv_bytes_read(self):
        """Same, counting each physical slot once (shared prefixes once)."""
        s = self.spec
        seen = set()
        B = self.block_size
        for i, n in enumerate(self.seq_lens.tolist()):
            nb = _nblocks(n, B)
            for j in range(nb):
                rows = min(B, n - j * B)
                blk = int(self.block_tables[i, j])
                for r in range(rows):
                    seen.add(blk * B + r)
        return len(seen) * 2 * s.num_kv_heads * s.head_dim * 2


def _build_metadata(spec, B, seed):
    rng = np.random.default_rng(seed)
    N = spec.num_seqs
    groups, gsize = spec.shared_groups, spec.shared_group_size
    n_shared = groups * gsize
    indep = _draw_lengths(spec.lengths, N - n_shared, rng)
    r = rng.integers(1, B, size=groups) if groups else np.zeros(0, np.int64)
    in_use = sum(_nblocks(n, B) for n in indep.tolist())
    for g in range(groups):
        in_use += _nblocks(spec.shared_prefix + int(r[g]), B) + (gsize - 1)
    NB = spec.fixed_num_blocks or int(math.ceil(spec.pool_factor * in_use))
    if NB < in_use:
        raise ValueError("pool too small for the workload")
    free = rng.permutation(NB).tolist()
    order = rng.permutation(N) if groups else np.arange(N)
    cursor = 0

    def take(k):
        nonlocal cursor
        out = free[cursor:cursor + k]
        cursor += k
        return out

    tables = [None] * N
    lens = np.zeros(N, np.int64)
    slots = np.zeros(N, np.int64)
    live = np.zeros((NB, B), dtype=bool)
    pairs = []
    # shared groups first (batch positions order[0 : n_shared])
    for g in range(groups):
        cached = spec.shared_prefix + int(r[g])
        base = take(_nblocks(cached, B))
        for j, blk in enumerate(base):
            live[blk, :min(B, cached - j * B)] = True
        for w in range(gsize):
            pos = int(order[g * gsize + w])
            if w < gsize - 1:
                fresh = take(1)[0]
                pairs.append((base[-1], fresh))
                tab = base[:-1] + [fresh]
            else:
                tab = list(base)
            tables[pos] = tab
            lens[pos] = cached + 1
            slots[pos] = tab[-1] * B + (cached - (len(tab) - 1) * B)
    for k, n in enumerate(indep.tolist()):
        pos = int(order[n_shared + k])
        tab = take(_nblocks(n, B))
        cached = n - 1
        for j, blk in enumerate(tab):
            live[blk, :max(0, min(B, cached - j * B))] = True
        tables[pos] = tab
        lens[pos] = n
        slots[pos] = tab[-1] * B + (cached - (len(tab) - 1) * B)
    maxb = max(len(t) for t in tables)
    bt = np.full((N, maxb), -1, dtype=np.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    cp = np.array(pairs, dtype=np.int32).reshape(-1, 2)
    return NB, lens.astype(np.int32), bt, slots, cp, live, np.array(free), np.asarray(order)


def _randn_bf16(shape, gen, device):
    return torch.randn(shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def make_workload(key_or_spec, block_size=None, seed=None, device="cpu", values=True,
                  poison=True, layers=None):
    """Build a workload.

    ``key_or_spec``: a config key (``tiny``, ``llama1b_layer``,
    ``continuous_batch``, ``long_context``, ``full_step``) or a spec.
    ``block_size`` overrides the spec's (the full-step sweep).  ``seed``
    overrides the spec's seed (multi-rank batches use ``rank_seed``).
    ``values=False`` builds metadata only.  ``layers`` limits how many layers
    of values are drawn (metadata is the same for every layer).
    """
    spec = get_spec(key_or_spec) if isinstance(key_or_spec, str) else key_or_spec
    B = int(block_size or spec.block_size)
    seed = spec.seed if seed is None else int(seed)
    NB, lens, bt, slots, cp, live, free, order = _build_metadata(spec, B, seed)
    w = Workload(spec=spec, block_size=B, num_blocks=NB, seq_lens=lens, block_tables=bt,
                 slot_mapping=slots, copy_pairs=cp, live_before=live, free_order=free,
                 batch_order=order, seed=seed)
    if not values:
        return w
    L = spec.num_layers if layers is None else int(layers)
    N, Hq, Hkv, d = w.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(seed)
    w.q = _randn_bf16((L, N, Hq, d), gen, dev)
    w.k_new = _randn_bf16((L, N, Hkv, d), gen, dev)
    w.v_new = _randn_bf16((L, N, Hkv, d), gen, dev)
    w.k_pool = torch.empty((L, NB, Hkv, B, d), dtype=torch.bfloat16, device=dev)
    w.v_pool = torch.empty((L, NB, Hkv, B, d), dtype=torch.bfloat16, device=dev)
    dead = torch.from_numpy(~live).to(dev)[:, None, :, None] if poison else None
    nan_bits = torch.tensor(BF16_NAN_BITS, dtype=torch.int16).view(torch.bfloat16).item()
    for layer in range(L):
        for pool in (w.k_pool, w.v_pool):
            pool[layer] = _randn_bf16((NB, Hkv, B, d), gen, dev)
            if poison:
                pool[layer].masked_fill_(dead, nan_bits)
    return w


def token_ids(w, vocab=128256, seed=None):
    """Token id of every position of every sequence, int32 ``[N, max_blocks*B]``
    (zero past each length), for the prefix-hash workload.

    Ids are drawn per physical slot (uniform over a Llama-3-sized vocabulary)
    and read through each sequence's table, so sequences that share a physical
    block share its tokens, as a shared prompt does.  A copy-on-write
    destination holds its source's tokens; each appended token gets its own id.
    Input generation only.
    """
    rng = np.random.default_rng(w.seed + 1000 if seed is None else seed)
    B = w.block_size
    slot_tok = rng.integers(0, vocab, w.num_blocks * B).astype(np.int32)
    for src, dst in w.copy_pairs.tolist():
        slot_tok[dst * B:(dst + 1) * B] = slot_tok[src * B:(src + 1) * B]
    slot_tok[w.slot_mapping] = rng.integers(0, vocab, w.num_seqs).astype(np.int32)
    N, maxb = w.block_tables.shape
    out = np.zeros((N, maxb * B), np.int32)
    for s in range(N):
        n = int(w.seq_lens[s])
        pos = np.arange(n)
        out[s, :n] = slot_tok[w.block_tables[s, pos // B].astype(np.int64) * B + pos % B]
    return out

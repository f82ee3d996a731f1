"""kv_append, block_copy and paged decode attention, in plain fp64 (oracle).

TEST INFRASTRUCTURE ONLY.

Layout (the library's contract; the pages fix no layout): a KV pool is an
array of bf16 bit patterns ``[num_blocks, num_kv_heads, block_size,
head_dim]`` per layer (``[num_layers, ...]`` for several layers); slot ``s``
is block ``s // B``, offset ``s % B``.

What is computed, restated from the pages:

* The attention formula is unchanged by paging: the kernel reads the
  sequence's K and V through the block table instead of from one contiguous
  range ([ITHOME] "PagedAttention 的核心想法"; [PU] "Continuous Batching",
  last paragraph: paging keeps dense attention semantics).
* Score of token i for query q: ``s_i = q . k_i / sqrt(d)``, softmax over
  every token the query can see, not per block ([PU] "按 Block 分配").  The
  ``1/sqrt(d)`` factor is passed in as ``scale``.
* Per block (or any computation partition) r: ``Z_r`` = sum of ``e^{s_i}``
  over its tokens, ``o_r`` = that block's own softmax output; the global
  output is ``(Z_1 o_1 + Z_2 o_2) / (Z_1 + Z_2)``, and more blocks merge the
  same way.  Each block's max score is recorded and the local sums are
  rescaled to a common base so that ``e^{s_i}`` cannot overflow; partitions
  need not coincide with physical blocks ([PU] "按 Block 分配", the merge
  equation, the 3 : 1 -> 0.75 / 0.25 example and the paragraph after it).
* Grouped-query attention: the pages name a GQA cache but not the head
  mapping; query head ``h`` reads kv head ``h // G`` with ``G = H_q / H_kv``
  (contiguous groups, the plainest reading).
* The token appended this step is attended to: lengths are post-append.

The main path (``paged_decode_attention``) is the plain max-subtracted
definition over the gathered tokens, i.e. the merge formula with a single
partition.  ``partial`` and ``merge`` implement the page's per-partition rule
and serve the split-K checks (``paged_decode_attention_split``).
"""

import numpy as np

from . import bf16 as _bf16
from .paging import translate


# --------------------------------------------------------------------------
# data movement (bit exact, on uint16 patterns)
# --------------------------------------------------------------------------

def kv_append(k_pool, v_pool, k_new, v_new, slot_mapping, block_size):
    """Write each new token's K and V (every kv head) into its slot.

    ``k_pool``/``v_pool``: uint16 ``[NB, H_kv, B, d]`` (one layer).
    ``k_new``/``v_new``: uint16 ``[T, H_kv, d]``; ``slot_mapping``: int ``[T]``,
    a negative slot means "padding, skip".  Returns new pools (inputs are not
    modified).  [ITHOME] "手動畫一次 block table": a new token goes into the
    next free slot of the tail block; [PU] "按 Block 分配": slot = (block,
    offset).
    """
    kp = _bf16.as_u16(k_pool).copy()
    vp = _bf16.as_u16(v_pool).copy()
    kn = _bf16.as_u16(k_new)
    vn = _bf16.as_u16(v_new)
    num_blocks = kp.shape[0]
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        blk, off = slot // block_size, slot % block_size
        if blk >= num_blocks:
            raise IndexError(f"slot {slot} outside the pool")
        for h in range(kp.shape[1]):
            kp[blk, h, off, :] = kn[t, h, :]
            vp[blk, h, off, :] = vn[t, h, :]
    return kp, vp


def block_copy(k_pools, v_pools, src_dst_pairs):
    """Copy whole blocks (every layer, every head, K and V): ``pool[l][dst] = pool[l][src]``.

    ``k_pools``/``v_pools``: uint16 ``[L, NB, H_kv, B, d]``.  Pairs are applied
    in order.  [PU] "共享前缀，分叉时 Copy-on-write": the writer's shared tail
    block is copied before it appends.
    """
    kp = _bf16.as_u16(k_pools).copy()
    vp = _bf16.as_u16(v_pools).copy()
    for src, dst in np.asarray(src_dst_pairs).reshape(-1, 2).tolist():
        for layer in range(kp.shape[0]):
            kp[layer, dst] = kp[layer, src]
            vp[layer, dst] = vp[layer, src]
    return kp, vp


def swap_blocks(src_k, src_v, dst_k, dst_v, src_dst_pairs):
    """Move whole blocks (every layer, every head, K and V) from one pool to
    another, e.g. device pool -> host pool when memory runs short and back:
    ``dst[l][d] = src[l][s]`` for each pair (s, d).  [AKIRA] 故事沒有說完的部分:
    under memory pressure blocks can be swapped out to CPU memory and brought
    back later.  Returns the new destination pools; the source is unchanged.
    """
    sk, sv = _bf16.as_u16(src_k), _bf16.as_u16(src_v)
    dk = _bf16.as_u16(dst_k).copy()
    dv = _bf16.as_u16(dst_v).copy()
    for src, dst in np.asarray(src_dst_pairs).reshape(-1, 2).tolist():
        for layer in range(dk.shape[0]):
            dk[layer, dst] = sk[layer, src]
            dv[layer, dst] = sv[layer, src]
    return dk, dv


# --------------------------------------------------------------------------
# attention
# --------------------------------------------------------------------------

def gather_tokens(pool, block_table, positions, block_size, kv_head):
    """Rows ``[len(positions), d]`` (float64) read position by position through the table.

    Each position is translated on its own (``translate``); the rows are then
    fetched with one fancy-index read of the pool.
    """
    where = [translate(block_table, p, block_size) for p in positions]
    d = pool.shape[-1]
    if not where:
        return np.zeros((0, d), dtype=np.float64)
    phys = np.array([w[0] for w in where], dtype=np.int64)
    off = np.array([w[1] for w in where], dtype=np.int64)
    if phys.min() < 0 or phys.max() >= pool.shape[0]:
        raise IndexError("block table entry outside the pool")
    return _bf16.to_f64(pool[phys, kv_head, off, :])


def softmax_attention(q, K, V, scale):
    """Dense single-query attention in fp64: max-subtracted softmax.

    ``q [d]``, ``K [n, d]``, ``V [n, d]``.  Returns ``o [d]``; an empty K
    gives zeros (nothing to attend to).
    """
    if K.shape[0] == 0:
        return np.zeros(V.shape[1], dtype=np.float64)
    s = scale * (K @ q)
    m = s.max()
    w = np.exp(s - m)
    return (w @ V) / w.sum()


def partial(q, K, V, scale):
    """One partition's statistics ``(m_r, Z_r, o_r)``.

    ``m_r`` = max score, ``Z_r`` = sum of ``e^{s_i - m_r}`` (the page's
    ``Z_r`` rescaled to base ``m_r``), ``o_r`` = the partition's own softmax
    output.  An empty partition returns ``(-inf, 0, zeros)``.
    """
    d = V.shape[1]
    if K.shape[0] == 0:
        return -np.inf, 0.0, np.zeros(d, dtype=np.float64)
    s = scale * (K @ q)
    m = s.max()
    w = np.exp(s - m)
    Z = w.sum()
    return m, Z, (w @ V) / Z


def merge(partials):
    """Max-rescaled merge ``o = sum_r e^{m_r-M} Z_r o_r / sum_r e^{m_r-M} Z_r``.

    [PU] "按 Block 分配": ``o = (Z_1 o_1 + Z_2 o_2) / (Z_1 + Z_2)`` with each
    ``Z_r`` brought to the common base ``M = max_r m_r``.  Returns
    ``(M, Z, o)`` so merges can be chained ("step by step or in parallel").
    """
    partials = list(partials)
    if not partials:
        raise ValueError("nothing to merge")
    M = max(p[0] for p in partials)
    d = len(partials[0][2])
    if M == -np.inf:
        return -np.inf, 0.0, np.zeros(d, dtype=np.float64)
    num = np.zeros(d, dtype=np.float64)
    den = 0.0
    for m, Z, o in partials:
        if Z == 0.0:
            continue
        c = np.exp(m - M) * Z
        num += c * np.asarray(o, dtype=np.float64)
        den += c
    return M, den, num / den


def _check_shapes(q, k_pool, v_pool, block_tables, seq_lens, block_size):
    q = _bf16.as_u16(q)
    k_pool = _bf16.as_u16(k_pool)
    v_pool = _bf16.as_u16(v_pool)
    N, Hq, d = q.shape
    NB, Hkv, B, d2 = k_pool.shape
    if B != block_size or d2 != d or v_pool.shape != k_pool.shape:
        raise ValueError("pool / query shape mismatch")
    if Hq % Hkv:
        raise ValueError("num_q_heads must be a multiple of num_kv_heads")
    if len(seq_lens) != N or len(block_tables) != N:
        raise ValueError("one block table and one length per sequence")
    return q, k_pool, v_pool, N, Hq, Hkv, d


def paged_decode_attention(q, k_pool, v_pool, block_tables, seq_lens, block_size, scale):
    """Decode-step attention through block tables, fp64, one output per query head.

    ``q`` uint16 ``[N, H_q, d]``; pools uint16 ``[NB, H_kv, B, d]``;
    ``block_tables`` ``[N, max_blocks]`` (entries past ``ceil(len/B)`` are
    never read); ``seq_lens`` ``[N]``.  Returns float64 ``[N, H_q, d]``.
    """
    q, k_pool, v_pool, N, Hq, Hkv, d = _check_shapes(
        q, k_pool, v_pool, block_tables, seq_lens, block_size)
    G = Hq // Hkv
    out = np.zeros((N, Hq, d), dtype=np.float64)
    for s in range(N):
        n = int(seq_lens[s])
        table = [int(x) for x in np.asarray(block_tables[s]).tolist()]
        for g in range(Hkv):
            K = gather_tokens(k_pool, table, range(n), block_size, g)
            V = gather_tokens(v_pool, table, range(n), block_size, g)
            for h in range(g * G, (g + 1) * G):
                out[s, h] = softmax_attention(_bf16.to_f64(q[s, h]), K, V, scale)
    return out


def paged_decode_attention_split(q, k_pool, v_pool, block_tables, seq_lens,
                                 block_size, scale, partition_tokens):
    """Same result via per-partition partials and the max-rescaled merge."""
    if partition_tokens <= 0:
        raise ValueError("partition_tokens must be positive")
    q, k_pool, v_pool, N, Hq, Hkv, d = _check_shapes(
        q, k_pool, v_pool, block_tables, seq_lens, block_size)
    G = Hq // Hkv
    out = np.zeros((N, Hq, d), dtype=np.float64)
    for s in range(N):
        n = int(seq_lens[s])
        table = [int(x) for x in np.asarray(block_tables[s]).tolist()]
        for g in range(Hkv):
            K = gather_tokens(k_pool, table, range(n), block_size, g)
            V = gather_tokens(v_pool, table, range(n), block_size, g)
            for h in range(g * G, (g + 1) * G):
                qh = _bf16.to_f64(q[s, h])
                parts = [partial(qh, K[a:a + partition_tokens], V[a:a + partition_tokens], scale)
                         for a in range(0, n, partition_tokens)]
                out[s, h] = merge(parts)[2] if parts else np.zeros(d)
    return out


def attention_rows(q, k_pool, v_pool, block_table, seq_len, block_size, scale, seq_index, heads):
    """Oracle output for a few (sequence, query head) pairs only.

    Used to check large workloads on sampled outputs: the same definition as
    ``paged_decode_attention`` restricted to one sequence and the listed
    query heads.  ``q`` is uint16 ``[N, H_q, d]``.
    """
    q = _bf16.as_u16(q)
    k_pool = _bf16.as_u16(k_pool)
    v_pool = _bf16.as_u16(v_pool)
    Hq = q.shape[1]
    Hkv = k_pool.shape[1]
    G = Hq // Hkv
    table = [int(x) for x in np.asarray(block_table).tolist()]
    res = {}
    cache = {}
    for h in heads:
        g = h // G
        if g not in cache:
            cache[g] = (gather_tokens(k_pool, table, range(seq_len), block_size, g),
                        gather_tokens(v_pool, table, range(seq_len), block_size, g))
        K, V = cache[g]
        res[h] = softmax_attention(_bf16.to_f64(q[seq_index, h]), K, V, scale)
    return res

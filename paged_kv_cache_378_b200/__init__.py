"""Paged KV-cache decode path for B200 (sm_100a): thin Python binding.

Every function here only checks and marshals arguments (torch CUDA tensors
-> raw device pointers + sizes + the current CUDA stream) and calls the C ABI
of ``libpagedkv.so`` (``include/pagedkv.h``); all work runs in the library's
CUDA kernels.  There is no CPU path: without the library, calls raise.

Names follow the pages' statement of the problem:

* ``kv_append(k, v, slot_mapping, k_pool, v_pool)`` -- new tokens fill their
  slots ("Infra: PagedAttention", section 按 Block 分配).
* ``paged_decode_attention(q, k_pool, v_pool, block_tables, seq_lens,
  block_size, scale, out)`` -- attention read through block tables, split
  into partitions merged by the max-rescaled rule (same section).
* ``block_copy(src_dst_pairs, k_pool, v_pool)`` -- copy-on-write of shared
  tail blocks (section 共享前缀，分叉时 Copy-on-write).

Pool tensors are bf16 ``[num_layers, num_blocks, num_kv_heads, block_size,
head_dim]`` (or without the leading layer dimension for one layer).
"""

import ctypes

import torch

from . import _lib
from ._lib import PkvBlockState, PkvCache

__all__ = [
    "PagedKVError", "kv_append", "block_copy", "paged_decode_attention",
    "append_paged_decode_attention", "BlockState", "block_manager_step", "block_manager_release",
    "swap_blocks",
    "SWAP_OUT", "SWAP_IN", "prefix_block_hashes",
    "attention_workspace_bytes", "partition_tokens", "make_workspace",
    "get_device_status", "set_wait_limit_ns", "workspace_init", "library", "DEV_RANGE",
    "DEV_LENGTH", "DEV_TIMEOUT", "DEV_NOBLOCKS", "COW_NO_APPEND",
]

DEV_RANGE = 0x1
DEV_LENGTH = 0x2
DEV_TIMEOUT = 0x4
DEV_NOBLOCKS = 0x8
COW_NO_APPEND = -2      # cow_src entry: the sequence appends nothing this step


class PagedKVError(RuntimeError):
    def __init__(self, code, where):
        self.code = code
        msg = library().pkv_strerror(code).decode()
        super().__init__(f"{where}: {msg} (status {code})")


def library():
    return _lib.load()


def _check(rc, where):
    if rc != 0:
        raise PagedKVError(rc, where)


def _need(t, name, dtype, device=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _pool_dims(k_pool, v_pool):
    _need(k_pool, "k_pool", torch.bfloat16)
    _need(v_pool, "v_pool", torch.bfloat16, k_pool.device)
    if k_pool.shape != v_pool.shape:
        raise ValueError("k_pool and v_pool shapes differ")
    if k_pool.dim() == 4:
        L = 1
        NB, H, B, D = k_pool.shape
    elif k_pool.dim() == 5:
        L, NB, H, B, D = k_pool.shape
    else:
        raise ValueError("pools must be [L, NB, H_kv, B, d] or [NB, H_kv, B, d]")
    return L, NB, H, B, D


def _cache(k_pool, v_pool):
    L, NB, H, B, D = _pool_dims(k_pool, v_pool)
    c = PkvCache(k_pool.data_ptr(), v_pool.data_ptr(), L, NB, H, B, D)
    return c, (L, NB, H, B, D)


def _stream(device, stream):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def kv_append(k, v, slot_mapping, k_pool, v_pool, layer=0, stream=None):
    """Store new tokens' K/V (bf16 ``[T, H_kv, d]``) at ``slot_mapping`` (int64 ``[T]``).

    ``slot < 0`` skips the token (padding).  Bit-exact copy.
    """
    cache, (L, NB, H, B, D) = _cache(k_pool, v_pool)
    dev = k_pool.device
    _need(k, "k", torch.bfloat16, dev)
    _need(v, "v", torch.bfloat16, dev)
    _need(slot_mapping, "slot_mapping", torch.int64, dev)
    T = slot_mapping.numel()
    if k.shape != (T, H, D) or v.shape != (T, H, D):
        raise ValueError(f"k/v must be [{T}, {H}, {D}]")
    rc = library().pkv_kv_append(ctypes.byref(cache), int(layer), k.data_ptr(), v.data_ptr(),
                                 slot_mapping.data_ptr(), T, _stream(dev, stream))
    _check(rc, "kv_append")


def block_copy(src_dst_pairs, k_pool, v_pool, num_pairs=None, stream=None):
    """Copy whole blocks (every layer, K and V): ``pool[:, dst] = pool[:, src]``.

    ``src_dst_pairs``: int32 ``[n, 2]``.  ``num_pairs``: optional int32 CUDA
    tensor ``[1]`` holding how many of the ``n`` pairs to copy (read on the
    device, e.g. the count ``block_manager_step`` wrote).
    """
    cache, _ = _cache(k_pool, v_pool)
    dev = k_pool.device
    _need(src_dst_pairs, "src_dst_pairs", torch.int32, dev)
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [n, 2]")
    n = src_dst_pairs.shape[0]
    if num_pairs is None:
        rc = library().pkv_block_copy(ctypes.byref(cache), src_dst_pairs.data_ptr(), n,
                                      _stream(dev, stream))
    else:
        _need(num_pairs, "num_pairs", torch.int32, dev)
        rc = library().pkv_block_copy_device_count(ctypes.byref(cache), src_dst_pairs.data_ptr(),
                                                   n, num_pairs.data_ptr(), _stream(dev, stream))
    _check(rc, "block_copy")


def prefix_block_hashes(tokens, seq_lens, block_size, extra_keys=None, max_blocks=None,
                        first_block=None, parent_hashes=None, out=None, stream=None):
    """Hash of every full block of every sequence (FNV-1a 64 chain over the
    parent hash, the block's tokens and the sequence's extra key).

    ``tokens`` int32 CUDA ``[N, T]``; ``seq_lens`` int32 ``[N]``; ``extra_keys``
    int64 ``[N]`` (bit patterns of uint64) or None.  Returns int64 ``[N,
    max_blocks]`` holding the uint64 bit patterns.  ``first_block`` (int32
    ``[N]``) and ``parent_hashes`` (int64 ``[N]``, the hash of block
    first_block - 1) resume a sequence's chain, e.g. for only the block that
    just became full; ``out`` receives the hashes in place (entries outside
    the hashed blocks keep their values; a fresh output starts at zero)."""
    dev = tokens.device
    _need(tokens, "tokens", torch.int32, dev)
    _need(seq_lens, "seq_lens", torch.int32, dev)
    if tokens.dim() != 2 or seq_lens.shape != (tokens.shape[0],):
        raise ValueError("tokens must be [N, T] and seq_lens [N]")
    N, T = tokens.shape
    if extra_keys is not None:
        _need(extra_keys, "extra_keys", torch.int64, dev)
        if extra_keys.shape != (N,):
            raise ValueError("extra_keys must be [N]")
    mb = T // int(block_size) if max_blocks is None else int(max_blocks)
    ptrs = []
    for t, name, dt in ((first_block, "first_block", torch.int32),
                        (parent_hashes, "parent_hashes", torch.int64)):
        if t is not None:
            _need(t, name, dt, dev)
            if t.shape != (N,):
                raise ValueError(f"{name} must be [N]")
        ptrs.append(t.data_ptr() if t is not None else None)
    if first_block is not None and parent_hashes is None:
        raise ValueError("first_block needs parent_hashes (the stored hash of the block "
                         "before each sequence's first one)")
    if out is None:
        out = torch.zeros((N, max(mb, 1)), dtype=torch.int64, device=dev)
    else:
        _need(out, "out", torch.int64, dev)
        if out.dim() != 2 or out.shape[0] != N or out.shape[1] != max(mb, 1):
            raise ValueError(f"out must be [N, {max(mb, 1)}] (max_blocks columns)")
    rc = library().pkv_prefix_block_hashes(
        tokens.data_ptr(), T, seq_lens.data_ptr(),
        extra_keys.data_ptr() if extra_keys is not None else None, ptrs[0], ptrs[1], N,
        int(block_size), out.data_ptr(), mb, _stream(dev, stream))
    _check(rc, "prefix_block_hashes")
    return out[:, :mb]


SWAP_OUT = 0
SWAP_IN = 1


def swap_blocks(src_dst_pairs, k_pool, v_pool, host_k_pool, host_v_pool, direction, stream=None):
    """Move whole blocks (every layer, K and V) between the device pools and
    pools in pinned host memory (``tensor.pin_memory()``), same shapes except
    the block count.  ``direction``: ``SWAP_OUT`` (host[dst] = device[src]) or
    ``SWAP_IN`` (device[dst] = host[src]); ``src_dst_pairs`` int32 CUDA ``[n, 2]``."""
    cache, _ = _cache(k_pool, v_pool)
    for t, name in ((host_k_pool, "host_k_pool"), (host_v_pool, "host_v_pool")):
        if not isinstance(t, torch.Tensor) or t.dtype != torch.bfloat16 or t.is_cuda \
                or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor in pinned memory")
        if not t.is_pinned():
            raise ValueError(f"{name} must be pinned (tensor.pin_memory())")
    if host_k_pool.shape != host_v_pool.shape:
        raise ValueError("host_k_pool and host_v_pool must have the same shape")
    L, NB, H, B, D = host_k_pool.shape
    host = PkvCache(host_k_pool.data_ptr(), host_v_pool.data_ptr(), L, NB, H, B, D)
    dev = k_pool.device
    _need(src_dst_pairs, "src_dst_pairs", torch.int32, dev)
    if src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be [n, 2]")
    rc = library().pkv_swap_blocks(ctypes.byref(cache), ctypes.byref(host), src_dst_pairs.data_ptr(),
                                   src_dst_pairs.shape[0], int(direction), _stream(dev, stream))
    _check(rc, "swap_blocks")


class BlockState:
    """Block manager state on the device: tables ``[N, max_blocks]``, lengths
    ``[N]``, reference counts ``[num_blocks]``, the free ring ``[num_blocks]``
    and ``free_state = [head, count]`` (all int32 CUDA tensors)."""

    def __init__(self, block_tables, seq_lens, refcount, free_ring, free_state):
        dev = block_tables.device
        for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens"),
                        (refcount, "refcount"), (free_ring, "free_ring"),
                        (free_state, "free_state")):
            _need(t, name, torch.int32, dev)
        if block_tables.dim() != 2 or seq_lens.shape != (block_tables.shape[0],):
            raise ValueError("block_tables must be [N, max_blocks] and seq_lens [N]")
        if refcount.dim() != 1 or free_ring.shape != refcount.shape or free_state.shape != (2,):
            raise ValueError("refcount and free_ring must be [num_blocks], free_state [2]")
        self.block_tables, self.seq_lens = block_tables, seq_lens
        self.refcount, self.free_ring, self.free_state = refcount, free_ring, free_state

    def _c(self):
        return PkvBlockState(self.block_tables.data_ptr(), self.seq_lens.data_ptr(),
                             self.refcount.data_ptr(), self.free_ring.data_ptr(),
                             self.free_state.data_ptr())


def block_manager_step(state, block_size, order=None, stream=None, with_cow_src=False):
    """One decode step of the block manager on the device (every sequence
    appends one token; ``order`` int32 ``[N]`` is the writer order).  Updates
    ``state`` in place; returns ``(slot_mapping int64 [N], copy_pairs int32
    [N, 2], num_pairs int32 [1])`` on the device, plus ``cow_src int32 [N]``
    (each sequence's copy source, -1 if none) with ``with_cow_src``."""
    dev = state.block_tables.device
    N, maxb = state.block_tables.shape
    nb = state.refcount.shape[0]
    if order is not None:
        _need(order, "order", torch.int32, dev)
        if order.shape != (N,):
            raise ValueError("order must be [N]")
    slots = torch.empty(N, dtype=torch.int64, device=dev)
    pairs = torch.empty((max(N, 1), 2), dtype=torch.int32, device=dev)
    npairs = torch.zeros(1, dtype=torch.int32, device=dev)
    cow = torch.empty(max(N, 1), dtype=torch.int32, device=dev)
    c = state._c()
    rc = library().pkv_block_manager_step(
        ctypes.byref(c), N, maxb, nb, int(block_size), order.data_ptr() if order is not None else None,
        slots.data_ptr(), pairs.data_ptr(), npairs.data_ptr(), cow.data_ptr(), _stream(dev, stream))
    _check(rc, "block_manager_step")
    if with_cow_src:
        return slots, pairs[:N], npairs, cow[:N]
    return slots, pairs[:N], npairs


def block_manager_release(state, block_size, seqs, stream=None):
    """Finished requests give their blocks back, on the device: ``seqs`` (int32
    ``[k]``, distinct rows) in order, each row's blocks in table order, lose a
    reference; blocks left with none join the free ring in that order; the
    rows' lengths become 0 and their tables -1.  Updates ``state`` in place."""
    dev = state.block_tables.device
    N, maxb = state.block_tables.shape
    nb = state.refcount.shape[0]
    _need(seqs, "seqs", torch.int32, dev)
    if seqs.dim() != 1:
        raise ValueError("seqs must be [k]")
    c = state._c()
    rc = library().pkv_block_manager_release(
        ctypes.byref(c), N, maxb, nb, int(block_size), seqs.data_ptr() if seqs.numel() else None,
        int(seqs.numel()), _stream(dev, stream))
    _check(rc, "block_manager_release")


def attention_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq,
                              block_size, partition_tokens=0):
    return int(library().pkv_attention_workspace_bytes(
        num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, block_size,
        partition_tokens))


def partition_tokens(num_seqs, num_kv_heads, head_dim, max_blocks_per_seq, block_size, requested=0):
    """Partition length the attention call will use (0 = library default)."""
    return int(library().pkv_partition_tokens(num_seqs, num_kv_heads, head_dim, max_blocks_per_seq,
                                              block_size, requested))


def make_workspace(num_seqs, num_q_heads, num_kv_heads, head_dim, max_blocks_per_seq, block_size,
                   partition_tokens=0, device="cuda"):
    """A zeroed workspace for these sizes (zeroed once; the kernel keeps it ready)."""
    n = attention_workspace_bytes(num_seqs, num_q_heads, num_kv_heads, head_dim,
                                  max_blocks_per_seq, block_size, partition_tokens)
    if n == 0:
        raise ValueError("invalid sizes for the attention workspace")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def paged_decode_attention(q, k_pool, v_pool, block_tables, seq_lens, block_size, scale, out,
                           layer=0, workspace=None, partition_tokens=0, stream=None):
    """Decode attention through block tables; writes bf16 ``out [N, H_q, d]``.

    ``q`` bf16 ``[N, H_q, d]``; ``block_tables`` int32 ``[N, max_blocks]``;
    ``seq_lens`` int32 ``[N]``; ``scale`` usually ``1/sqrt(d)``.
    ``workspace``: uint8 CUDA tensor from ``make_workspace`` (required when a
    sequence can span several partitions).
    """
    cache, (L, NB, H, B, D) = _cache(k_pool, v_pool)
    if int(block_size) != B:
        raise ValueError(f"block_size {block_size} does not match the pools ({B})")
    dev = k_pool.device
    _need(q, "q", torch.bfloat16, dev)
    _need(out, "out", torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(seq_lens, "seq_lens", torch.int32, dev)
    if q.dim() != 3 or q.shape[2] != D:
        raise ValueError(f"q must be [N, H_q, {D}]")
    N, Hq, _ = q.shape
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    if block_tables.dim() != 2 or block_tables.shape[0] != N or seq_lens.shape != (N,):
        raise ValueError("block_tables must be [N, max_blocks] and seq_lens [N]")
    maxb = block_tables.shape[1]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, dev)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
    rc = library().pkv_paged_decode_attention(
        ctypes.byref(cache), int(layer), q.data_ptr(), N, Hq, block_tables.data_ptr(), maxb,
        seq_lens.data_ptr(), float(scale), out.data_ptr(), ws_ptr, ws_bytes, int(partition_tokens),
        _stream(dev, stream))
    _check(rc, "paged_decode_attention")
    return out


def append_paged_decode_attention(k_new, v_new, q, k_pool, v_pool, block_tables, seq_lens,
                                  block_size, scale, out, layer=0, workspace=None,
                                  partition_tokens=0, cow_src=None, stream=None):
    """Fused decode step of one layer: store each sequence's newest token
    (``k_new``/``v_new`` bf16 ``[N, H_kv, d]``, position ``seq_lens[s] - 1``,
    slot from the block table) and attend over the updated cache; writes
    ``out``.  Same result as ``kv_append`` with that slot mapping followed by
    ``paged_decode_attention``.  ``cow_src`` (int32 ``[N]``, -1 = none): the
    tail block of sequence s is made here as a copy of block ``cow_src[s]``
    (this layer), as ``block_copy`` would before the append."""
    cache, (L, NB, H, B, D) = _cache(k_pool, v_pool)
    if int(block_size) != B:
        raise ValueError(f"block_size {block_size} does not match the pools ({B})")
    dev = k_pool.device
    for t, name in ((k_new, "k_new"), (v_new, "v_new"), (q, "q"), (out, "out")):
        _need(t, name, torch.bfloat16, dev)
    _need(block_tables, "block_tables", torch.int32, dev)
    _need(seq_lens, "seq_lens", torch.int32, dev)
    if q.dim() != 3 or q.shape[2] != D:
        raise ValueError(f"q must be [N, H_q, {D}]")
    N, Hq, _ = q.shape
    if k_new.shape != (N, H, D) or v_new.shape != (N, H, D):
        raise ValueError(f"k_new and v_new must be [N, {H}, {D}]")
    if out.shape != q.shape:
        raise ValueError("out must have q's shape")
    if block_tables.dim() != 2 or block_tables.shape[0] != N or seq_lens.shape != (N,):
        raise ValueError("block_tables must be [N, max_blocks] and seq_lens [N]")
    maxb = block_tables.shape[1]
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        _need(workspace, "workspace", torch.uint8, dev)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel()
    cow_ptr = None
    if cow_src is not None:
        _need(cow_src, "cow_src", torch.int32, dev)
        if cow_src.shape != (N,):
            raise ValueError("cow_src must be [N]")
        cow_ptr = cow_src.data_ptr()
    rc = library().pkv_append_paged_decode_attention(
        ctypes.byref(cache), int(layer), k_new.data_ptr(), v_new.data_ptr(), cow_ptr, q.data_ptr(), N, Hq,
        block_tables.data_ptr(), maxb, seq_lens.data_ptr(), float(scale), out.data_ptr(), ws_ptr,
        ws_bytes, int(partition_tokens), _stream(dev, stream))
    _check(rc, "append_paged_decode_attention")
    return out


def set_wait_limit_ns(limit_ns=0):
    """Limit (ns) of the attention kernel's bounded wait for a staged tile on
    the current device; 0 restores the default (2 s).  A launch whose wait
    runs out sets DEV_TIMEOUT; zero its workspace again afterwards."""
    _check(library().pkv_set_wait_limit_ns(int(limit_ns)), "set_wait_limit_ns")


def workspace_init(workspace, stream=None):
    """Zero an attention workspace again (after a launch that timed out)."""
    _need(workspace, "workspace", torch.uint8)
    _check(library().pkv_workspace_init(workspace.data_ptr(), workspace.numel(),
                                        _stream(workspace.device, stream)), "workspace_init")


def get_device_status(reset=True):
    """Device status bits (DEV_RANGE | DEV_LENGTH | DEV_TIMEOUT); synchronises the device."""
    v = ctypes.c_uint(0)
    _check(library().pkv_get_device_status(ctypes.byref(v), 1 if reset else 0), "get_device_status")
    return int(v.value)

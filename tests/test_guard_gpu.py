"""Guard regions around every buffer the kernels write (the pools, the output
and the attention workspace): each sits in the middle of a larger buffer whose
head and tail hold a sentinel bit pattern.  After the fused copy-on-write +
append + attention step, the separate copy, append and attention calls, and
the no-allocation attention call, every guard must be untouched and every
result must equal the same calls on ordinary tensors, bit for bit.  An
out-of-bounds write shows without a sanitizer and without faulting.
"""

import ctypes

import numpy as np
import pytest
import torch

from workload import make_workload
from workload.configs import WorkloadSpec

from .stepping import cow_sources

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import paged_kv_cache_378_b200 as pkv
else:  # collected on CPU-only machines, never run there
    pkv = None

GUARD = 4096                    # elements of guard on each side (16-byte multiples)
SENTINEL = 0x7FC1               # a bf16 NaN pattern nothing here writes


def _guarded(like, dtype=None):
    """A contiguous tensor shaped like `like` inside a sentinel-filled buffer."""
    dtype = dtype or like.dtype
    n = like.numel()
    buf = torch.empty(n + 2 * GUARD, dtype=torch.int16, device="cuda") if dtype == torch.bfloat16 \
        else torch.empty(n + 2 * GUARD, dtype=dtype, device="cuda")
    if dtype == torch.bfloat16:
        buf.fill_(SENTINEL)
        view = buf[GUARD:GUARD + n].view(torch.bfloat16).view(like.shape)
    else:
        buf.fill_(0x5A if dtype == torch.uint8 else SENTINEL)
        view = buf[GUARD:GUARD + n].view(like.shape)
    return buf, view


def _guards_intact(buf, what):
    fill = 0x5A if buf.dtype == torch.uint8 else SENTINEL
    head, tail = buf[:GUARD], buf[-GUARD:]
    assert bool((head == fill).all()) and bool((tail == fill).all()), f"{what}: a guard was written"


SPECS = [
    "continuous_batch",
    WorkloadSpec(key="guard_d128", title="d128, G=4, B=32", num_layers=2, num_seqs=40,
                 num_q_heads=16, num_kv_heads=4, head_dim=128, block_size=32, seed=21,
                 lengths="uniform:1,900"),
]


@pytest.mark.parametrize("key", SPECS, ids=["continuous_batch", "d128"])
@pytest.mark.parametrize("partition", [0, 64])
def test_no_write_outside_pools_output_and_workspace(key, partition):
    w = make_workload(key, poison=False)
    spec = w.spec
    dev = torch.device("cuda")
    q, k_new, v_new = w.q.to(dev), w.k_new.to(dev), w.v_new.to(dev)
    tables = torch.from_numpy(w.block_tables).to(dev)
    lens = torch.from_numpy(w.seq_lens).to(dev)
    slots = torch.from_numpy(w.slot_mapping).to(dev)
    pairs = torch.from_numpy(w.copy_pairs).to(dev)
    cow = torch.from_numpy(cow_sources(w)).to(dev)
    nbytes = pkv.attention_workspace_bytes(w.num_seqs, spec.num_q_heads, spec.num_kv_heads,
                                           spec.head_dim, w.max_blocks, w.block_size, partition)

    def run(guard):
        if guard:
            kb, kp = _guarded(w.k_pool)
            vb, vp = _guarded(w.v_pool)
            ob, out = _guarded(w.q[0])
            wb, ws = _guarded(torch.empty(nbytes, dtype=torch.uint8), torch.uint8)
        else:
            kp, vp = torch.empty_like(w.k_pool, device=dev), torch.empty_like(w.v_pool, device=dev)
            out = torch.empty_like(q[0])
            ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        kp.copy_(w.k_pool)
        vp.copy_(w.v_pool)
        pkv.workspace_init(ws)
        results = []
        for layer in range(spec.num_layers):
            pkv.append_paged_decode_attention(k_new[layer], v_new[layer], q[layer], kp, vp, tables,
                                              lens, w.block_size, spec.scale, out, layer=layer,
                                              workspace=ws, partition_tokens=partition,
                                              cow_src=cow)
            results.append(out.clone())
        # the separate calls on the same pools (copies and appends again: same values)
        pkv.block_copy(pairs, kp, vp)
        for layer in range(spec.num_layers):
            pkv.kv_append(k_new[layer], v_new[layer], slots, kp, vp, layer=layer)
            pkv.paged_decode_attention(q[layer], kp, vp, tables, lens, w.block_size, spec.scale,
                                       out, layer=layer, workspace=ws, partition_tokens=partition)
            results.append(out.clone())
        # the no-allocation attention call (its scratch is inside the library;
        # under the 64-token cap this batch needs more, which it refuses)
        from paged_kv_cache_378_b200._lib import PkvCache
        L, NB, H, B, D = kp.shape
        cache = PkvCache(kp.data_ptr(), vp.data_ptr(), L, NB, H, B, D)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for layer in range(spec.num_layers if partition == 0 else 0):
            rc = pkv.library().pkv_paged_decode_attention_noalloc(
                ctypes.byref(cache), layer, q[layer].data_ptr(), w.num_seqs, spec.num_q_heads,
                tables.data_ptr(), w.max_blocks, lens.data_ptr(), ctypes.c_float(spec.scale),
                out.data_ptr(), partition, stream)
            assert rc == 0, pkv.library().pkv_strerror(rc)
            results.append(out.clone())
        torch.cuda.synchronize()
        assert pkv.get_device_status(reset=True) == 0
        if guard:
            for b, what in ((kb, "K pool"), (vb, "V pool"), (ob, "output"), (wb, "workspace")):
                _guards_intact(b, what)
        return results, kp.clone(), vp.clone()

    pkv.get_device_status(reset=True)
    plain = run(False)
    guarded = run(True)
    for a, b in zip(plain[0], guarded[0]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(plain[1].view(torch.int16), guarded[1].view(torch.int16))
    assert torch.equal(plain[2].view(torch.int16), guarded[2].view(torch.int16))

"""pkv_paged_decode_attention_noalloc: the attention call for callers that
cannot allocate device memory (for example a plugin that is handed only its
input and output buffers, or a serving loop that must never call the
allocator).  Its scratch is a fixed array inside the library, so the call
needs no workspace.

Checked here through the C ABI: two calls in a row give the same output as
the workspace-taking entry point, within the parity tolerance, and a request
too large for the fixed scratch is refused before anything is launched.  The
file sorts last so that, if it fails, a run stopping at the first failure has
already run every other test; it passes alone in a fresh process too.
"""

import ctypes

import numpy as np
import pytest
import torch

from workload import make_workload
from workload.configs import WorkloadSpec

from .stepping import assert_close, f64

pytestmark = pytest.mark.gpu


# More than 768 sequences (the tile prefix then lives in the scratch too), the
# widest group (G = 8) at head_dim 128: the largest scratch of an uncapped call.
WIDE = WorkloadSpec(key="noalloc_wide", title="1000 seqs, G=8, d128", num_layers=1, num_seqs=1000,
                    num_q_heads=32, num_kv_heads=4, head_dim=128, block_size=16, seed=77,
                    lengths="uniform:1,300")


def _inputs(key, device):
    # no NaN poison: this test runs attention without the step's kv_append, so the
    # new token's slot must hold a value
    w = make_workload(key, poison=False)
    spec = w.spec
    kp = w.k_pool.to(device)
    vp = w.v_pool.to(device)
    q = w.q[0].to(device)
    tables = torch.from_numpy(w.block_tables).to(device)
    lens = torch.from_numpy(w.seq_lens).to(device)
    return w, spec, kp, vp, q, tables, lens


@pytest.mark.parametrize("key", ["continuous_batch", "long_context", WIDE])
def test_noalloc_matches_workspace_call_on_two_calls(key):
    import paged_kv_cache_378_b200 as pkv
    from paged_kv_cache_378_b200._lib import PkvCache

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    lib = pkv.library()
    w, spec, kp, vp, q, tables, lens = _inputs(key, dev)
    pkv.get_device_status(reset=True)

    # the existing entry point, with a caller-owned workspace
    ref = torch.empty_like(q)
    ws = pkv.make_workspace(w.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim,
                            w.max_blocks, w.block_size, 0, device=dev)
    # the scratch holds what the workspace-taking call needs for the same sizes
    assert ws.numel() <= 16 << 20, ws.numel()
    pkv.paged_decode_attention(q, kp, vp, tables, lens, w.block_size, spec.scale, ref, workspace=ws)
    torch.cuda.synchronize()

    L, NB, H, B, D = kp.shape
    cache = PkvCache(kp.data_ptr(), vp.data_ptr(), L, NB, H, B, D)
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    outs = []
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        rc = lib.pkv_paged_decode_attention_noalloc(
            ctypes.byref(cache), 0, q.data_ptr(), w.num_seqs, spec.num_q_heads, tables.data_ptr(),
            w.max_blocks, lens.data_ptr(), ctypes.c_float(spec.scale), out.data_ptr(), 0, stream)
        assert rc == 0, lib.pkv_strerror(rc)
        torch.cuda.synchronize()
        outs.append(out)
    assert pkv.get_device_status(reset=True) == 0
    want = f64(ref)
    assert np.all(np.isfinite(want))
    for i, out in enumerate(outs):
        name = key if isinstance(key, str) else key.key
        assert_close(f64(out), want, f"{name} no-alloc call {i}")
        # same kernel, same schedule: the same bits
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"{name} call {i}"


def test_noalloc_refuses_requests_larger_than_its_scratch():
    import paged_kv_cache_378_b200 as pkv
    from paged_kv_cache_378_b200._lib import PkvCache

    dev = torch.device("cuda", 0)
    lib = pkv.library()
    w, spec, kp, vp, q, tables, lens = _inputs("continuous_batch", dev)
    L, NB, H, B, D = kp.shape
    cache = PkvCache(kp.data_ptr(), vp.data_ptr(), L, NB, H, B, D)
    out = torch.zeros_like(q)
    # a 32-token partition cap splits the batch into far more ranges than 16 MiB holds
    rc = lib.pkv_paged_decode_attention_noalloc(
        ctypes.byref(cache), 0, q.data_ptr(), w.num_seqs, spec.num_q_heads, tables.data_ptr(),
        w.max_blocks, lens.data_ptr(), ctypes.c_float(spec.scale), out.data_ptr(), 32, None)
    assert rc == -8
    assert b"no-allocation" in lib.pkv_strerror(rc)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0        # nothing was launched

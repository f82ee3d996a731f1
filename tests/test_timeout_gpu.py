"""The attention kernel's bounded wait, driven to give up without any fault.

Every wait on a staged tile is bounded; when the limit runs out the warp sets
PKV_DEV_TIMEOUT, waits (with its own fixed limit) for the copies it has in
flight, and exits.  A limit of one nanosecond makes the first waits give up
while every load is still valid: nothing faults and nothing waits forever.
Afterwards the workspace is zeroed again, the default limit restored, and a
normal launch must match the oracle.
"""

import pytest
import torch

from oracle import attention as oa
from workload import make_workload

from .stepping import assert_close, device_inputs, f64, u16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import paged_kv_cache_378_b200 as pkv
else:  # collected on CPU-only machines, never run there
    pkv = None


def _attend(w, dev, ws, out):
    spec = w.spec
    pkv.paged_decode_attention(dev["q"][0], dev["k_pool"], dev["v_pool"], dev["tables"],
                               dev["lens"], w.block_size, spec.scale, out, layer=0, workspace=ws)


def test_bounded_wait_gives_up_and_the_device_stays_usable():
    w = make_workload("continuous_batch", poison=False)
    spec = w.spec
    dev = device_inputs(w)
    ws = pkv.make_workspace(w.num_seqs, spec.num_q_heads, spec.num_kv_heads, spec.head_dim,
                            w.max_blocks, w.block_size, 0)
    out = torch.empty_like(dev["q"][0])
    pkv.get_device_status(reset=True)
    pkv.set_wait_limit_ns(1)
    try:
        _attend(w, dev, ws, out)
        status = pkv.get_device_status(reset=True)      # synchronises: every warp has exited
    finally:
        pkv.set_wait_limit_ns(0)
    assert status & pkv.DEV_TIMEOUT, f"status {status:#x}"
    assert status & ~pkv.DEV_TIMEOUT == 0, f"status {status:#x}"
    # after a timeout the workspace's counters are undefined: zero it, then a
    # normal launch is exact again
    pkv.workspace_init(ws)
    _attend(w, dev, ws, out)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    ref = oa.paged_decode_attention(u16(w.q[0]), u16(w.k_pool[0]), u16(w.v_pool[0]),
                                    w.block_tables, w.seq_lens, w.block_size, spec.scale)
    assert_close(f64(out), ref, "after a timeout")

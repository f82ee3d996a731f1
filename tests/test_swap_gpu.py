"""GPU parity of block swap between the device pool and a pinned host pool
against the oracle's swap_blocks: bit exact in both directions."""

import numpy as np
import pytest
import torch

from oracle import attention as oa

from .stepping import u16

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import paged_kv_cache_378_b200 as pkv
else:  # collected on CPU-only machines, never run there
    pkv = None


@pytest.fixture(autouse=True)
def _clean_status():
    if torch.cuda.is_available():
        pkv.get_device_status(reset=True)
    yield


@pytest.mark.parametrize("L,H,B,D", [(2, 8, 16, 64), (3, 2, 4, 128), (1, 8, 32, 64)])
def test_swap_out_and_in_bit_exact(L, H, B, D):
    g = torch.Generator().manual_seed(L * 100 + B + D)
    NB, NH = 40, 24
    kp = torch.randn((L, NB, H, B, D), generator=g).to(torch.bfloat16)
    vp = torch.randn((L, NB, H, B, D), generator=g).to(torch.bfloat16)
    kp.view(torch.int16)[0, 3, 0, 0, :2] = torch.tensor([0x7FC1, -32768], dtype=torch.int16)
    hk = torch.zeros((L, NH, H, B, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.zeros_like(hk).pin_memory()
    kd, vd = kp.cuda(), vp.cuda()
    rng = np.random.default_rng(B + D)
    out = np.stack([rng.choice(NB, 12, replace=False), rng.choice(NH, 12, replace=False)], 1)
    pkv.swap_blocks(torch.from_numpy(out.astype(np.int32)).cuda(), kd, vd, hk, hv, pkv.SWAP_OUT)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    ek, ev = oa.swap_blocks(u16(kp), u16(vp), np.zeros(hk.shape, np.uint16),
                            np.zeros(hv.shape, np.uint16), out)
    assert np.array_equal(u16(hk), ek) and np.array_equal(u16(hv), ev)
    # back in, into other device blocks
    back = np.stack([out[:, 1], rng.choice(NB, 12, replace=False)], 1)
    host_k, host_v = u16(hk), u16(hv)
    pkv.swap_blocks(torch.from_numpy(back.astype(np.int32)).cuda(), kd, vd, hk, hv, pkv.SWAP_IN)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == 0
    ek2, ev2 = oa.swap_blocks(host_k, host_v, u16(kp), u16(vp), back)
    assert np.array_equal(u16(kd), ek2) and np.array_equal(u16(vd), ev2)


def test_swap_rejects_pageable_host_memory_and_reports_bad_ids():
    L, NB, H, B, D = 1, 8, 2, 16, 64
    kd = torch.zeros((L, NB, H, B, D), dtype=torch.bfloat16, device="cuda")
    vd = torch.zeros_like(kd)
    pairs = torch.tensor([[1, 2]], dtype=torch.int32, device="cuda")
    # pageable host pools are refused by the C library itself
    from paged_kv_cache_378_b200._lib import PkvCache
    import ctypes
    hk = torch.zeros((L, 4, H, B, D), dtype=torch.bfloat16)
    hv = torch.zeros_like(hk)
    dev = PkvCache(kd.data_ptr(), vd.data_ptr(), L, NB, H, B, D)
    host = PkvCache(hk.data_ptr(), hv.data_ptr(), L, 4, H, B, D)
    rc = pkv.library().pkv_swap_blocks(ctypes.byref(dev), ctypes.byref(host), pairs.data_ptr(), 1,
                                       0, None)
    assert rc == -9
    # a block id outside the host pool: skipped and reported, the context still works
    hk, hv = hk.pin_memory(), hv.pin_memory()
    bad = torch.tensor([[1, 4], [2, 3]], dtype=torch.int32, device="cuda")
    kd[:, 2] = 1.0
    pkv.swap_blocks(bad, kd, vd, hk, hv, pkv.SWAP_OUT)
    torch.cuda.synchronize()
    assert pkv.get_device_status(reset=True) == pkv.DEV_RANGE
    assert torch.all(hk[:, 3] == 1.0) and torch.all(hk[:, :3] == 0)

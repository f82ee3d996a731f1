"""Helpers shared by the GPU parity tests: run one decode step through the
C ABI binding, run the same step through the oracle, compare.

A decode step (per layer) is: copy-on-write block copies (once, all layers),
then for each layer kv_append of the new tokens, then paged decode attention.
"""

import numpy as np
import torch

from oracle import attention as oa
from oracle import bf16 as ob

ATOL = 1e-2
RTOL = 1e-2


def u16(t):
    """bf16 torch tensor (any device) -> numpy uint16 bit patterns (host copy)."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def f64(t):
    return ob.to_f64(u16(t))


def device_inputs(w, device="cuda"):
    """Move a workload's tensors and metadata to the GPU (pools are cloned)."""
    d = torch.device(device)
    return dict(
        k_pool=w.k_pool.to(d).clone(), v_pool=w.v_pool.to(d).clone(),
        q=w.q.to(d), k_new=w.k_new.to(d), v_new=w.v_new.to(d),
        tables=torch.from_numpy(w.block_tables).to(d),
        lens=torch.from_numpy(w.seq_lens).to(d),
        slots=torch.from_numpy(w.slot_mapping).to(d),
        pairs=torch.from_numpy(w.copy_pairs).to(d),
    )


def cow_sources(w):
    """Per sequence, the source block of this step's copy-on-write (-1 if
    none): the pair whose destination is the sequence's tail block."""
    src_of = {int(d): int(s) for s, d in w.copy_pairs}
    tails = w.block_tables[np.arange(w.num_seqs), (w.seq_lens.astype(np.int64) - 1) // w.block_size]
    return np.array([src_of.get(int(t), -1) for t in tails], np.int32)


def gpu_step(pkv, w, dev_in, layers=None, partition_tokens=None, workspace=None, fused=False,
             cow=False):
    """Run the step with the CUDA library; returns {layer: out bf16 tensor}.

    ``fused``: append and attention of each layer in one call
    (``append_paged_decode_attention``) instead of ``kv_append`` then
    ``paged_decode_attention``.  ``cow`` (with ``fused``): the copy-on-write is
    folded into those calls too (``cow_src``) instead of a ``block_copy``."""
    spec = w.spec
    part = spec.partition_tokens if partition_tokens is None else partition_tokens
    L = dev_in["k_pool"].shape[0]
    layers = range(L) if layers is None else layers
    if workspace is None:
        workspace = pkv.make_workspace(w.num_seqs, spec.num_q_heads, spec.num_kv_heads,
                                       spec.head_dim, w.max_blocks, w.block_size, part,
                                       device=dev_in["q"].device)
    cow_src = None
    if fused and cow:
        cow_src = torch.from_numpy(cow_sources(w)).to(dev_in["q"].device)
    else:
        pkv.block_copy(dev_in["pairs"], dev_in["k_pool"], dev_in["v_pool"])
    outs = {}
    for layer in layers:
        out = torch.empty_like(dev_in["q"][layer])
        if fused:
            pkv.append_paged_decode_attention(
                dev_in["k_new"][layer], dev_in["v_new"][layer], dev_in["q"][layer],
                dev_in["k_pool"], dev_in["v_pool"], dev_in["tables"], dev_in["lens"], w.block_size,
                spec.scale, out, layer=layer, workspace=workspace, partition_tokens=part,
                cow_src=cow_src)
            outs[layer] = out
            continue
        pkv.kv_append(dev_in["k_new"][layer], dev_in["v_new"][layer], dev_in["slots"],
                      dev_in["k_pool"], dev_in["v_pool"], layer=layer)
        pkv.paged_decode_attention(dev_in["q"][layer], dev_in["k_pool"], dev_in["v_pool"],
                                   dev_in["tables"], dev_in["lens"], w.block_size, spec.scale, out,
                                   layer=layer, workspace=workspace, partition_tokens=part)
        outs[layer] = out
    torch.cuda.synchronize()
    return outs


def oracle_pools_after_step(w, host_k, host_v, layer):
    """Oracle: block copies (all layers share the pairs) then kv_append, one layer."""
    kp, vp = oa.block_copy(host_k[None], host_v[None], w.copy_pairs)
    return oa.kv_append(kp[0], vp[0], u16(w.k_new[layer]), u16(w.v_new[layer]),
                        w.slot_mapping, w.block_size)


def assert_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = np.abs(got - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(f"{what}: {int(bad.sum())} elements outside |err| <= {ATOL} + {RTOL}|ref|;"
                             f" max err {err.max():.3e}; first {idx.tolist()}")
    return float(err.max())

"""Benchmark of the paged decode path (copy-on-write block copy + kv_append +
paged decode attention) on B200, one JSON line on stdout.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload KEY]
                    [--block-size B] [--partition P] [--impl ours|reference]

A step is one pass of the whole path over one batch: block_copy of the
batch's copy-on-write pairs (every layer), then for each layer kv_append of
one new token per sequence and paged decode attention.  Inputs are seeded
synthetic data of the workload's shapes (``workload/``), resident in HBM
before the timed region; L2 reuse across steps is prevented by rotating
through several copies of the KV pools whose total is over 4x the L2 size.

Multi-GPU (torchrun): every rank runs its own independent batch (weak
scaling, no data-path collective); the timed region is bracketed by a barrier
and the device time is the max over ranks.
"""

import argparse
import ctypes
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from workload import make_workload, rank_seed  # noqa: E402
from workload.configs import get_spec  # noqa: E402

METRIC = "paged decode attention KV GB/s and % of HBM peak; decode tokens/s per layer"
UNIT = "GB/s"
DEFAULT_WORKLOAD = "continuous_batch"
FALLBACK_HBM_GBS = 6650.0
SPIN_CYCLES = 4_000_000    # ~2 ms of spinning ahead of a timed region
NOMINAL_HBM_GBS = 8000.0   # the ~8 TB/s the 70 % bandwidth target is stated against
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "attention_traffic.json")
EVENT_EVERY = 8            # attention events on every 8th timed step
# device sources of the attention kernel: a committed DRAM-traffic capture
# stands only while these are unchanged
KERNEL_SOURCES = ["pkv_device.cuh", "attn_common.cuh", "attn_paged.cuh"]


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

def kernel_source_hash():
    """Hash of the attention kernel's device sources with comments and blank
    lines removed, so an edit to comments alone keeps a capture valid."""
    import re
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "paged_kv_cache_378_b200", "csrc", f), encoding="utf-8") as fh:
            text = fh.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        lines = [ln.split("//", 1)[0].rstrip() for ln in text.splitlines()]
        h.update("\n".join(ln for ln in lines if ln.strip()).encode())
    return h.hexdigest()[:16]


def load_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def load_traffic(workload_key, block_size, step, partition):
    """DRAM bytes per attention launch from the committed ncu summary, or None
    if absent, for another workload, step or partition cap, or taken on
    different kernel source."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    for r in rec.get("captures", []):
        if r.get("workload") == workload_key and int(r.get("block_size", -1)) == block_size \
                and r.get("step") == step \
                and int(r.get("partition_tokens", 0)) == partition \
                and r.get("kernel_source_hash") == kernel_source_hash():
            return r.get("dram_bytes_per_launch")
    return None


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons in the background."""

    FIELDS = ("index,pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, pci_bus_id=None, period_ms=100):
        self.pci = (pci_bus_id or "").strip().lower()
        self.period_ms = period_ms
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", str(self.period_ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL,
                text=True)
        except OSError:
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            if self.pci and not parts[1].lower().endswith(self.pci[-12:]):
                continue
            self.rows.append((time.time(), parts))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        rows = [r for t, r in self.rows if t0 <= t <= t1]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(r[2]) for r in rows if num(r[2]) is not None]
        mx = [num(r[3]) for r in rows if num(r[3]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows),
                "power_w_max": max((num(r[4]) or 0.0) for r in rows)}


def pci_bus_id(dev):
    try:
        from cuda.bindings import runtime as rt
        err, bus = rt.cudaDeviceGetPCIBusId(32, dev)
        if int(err) == 0:
            bus = bus.decode() if isinstance(bus, bytes) else str(bus)
            return bus.replace("\x00", "").strip()
    except Exception:
        pass
    return None


def gpu_local_cpus(bus):
    """CPUs on the GPU's own NUMA node (sysfs ``local_cpulist``), or None."""
    if not bus:
        return None
    dom, rest = bus.lower().split(":", 1)
    path = f"/sys/bus/pci/devices/{dom[-4:]}:{rest}/local_cpulist"
    try:
        text = open(path).read().strip()
    except OSError:
        return None
    cpus = set()
    for part in text.split(","):
        lo, _, hi = part.partition("-")
        cpus.update(range(int(lo), int(hi or lo) + 1))
    cpus &= os.sched_getaffinity(0)
    return cpus or None


def combine_over_ranks(dist, ms, nbytes, nseqs, device):
    """(max device ms, total bytes, total sequences) over all ranks.

    Every rank must call this the same number of times, in the same order.
    """
    if dist is None:
        return float(ms), float(nbytes), float(nseqs)
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    w = torch.tensor([nbytes, nseqs], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(w, op=dist.ReduceOp.SUM)
    return float(t[0]), float(w[0]), float(w[1])


# ---------------------------------------------------------------------------
# the GPU step through the C ABI
# ---------------------------------------------------------------------------

class GpuStep:
    """One decode step through the C ABI with arguments marshalled once.

    Calls the library's entry points directly (the same C functions the
    Python binding wraps), so per-step host overhead stays far below the
    device time of a step.
    """

    def __init__(self, pkv, w, replicas, partition, device, mode="cow"):
        from paged_kv_cache_378_b200._lib import PkvCache
        self.lib = pkv.library()
        spec = w.spec
        self.w = w
        self.L = spec.num_layers
        self.N = w.num_seqs
        self.Hq = spec.num_q_heads
        self.device = device
        self.stream = torch.cuda.current_stream(device)
        self.sp = ctypes.c_void_p(self.stream.cuda_stream)
        self.replicas = replicas
        self.caches = []
        L, NB, H, B, D = w.k_pool.shape
        for kp, vp in replicas:
            c = PkvCache(kp.data_ptr(), vp.data_ptr(), L, NB, H, B, D)
            self.caches.append((c, ctypes.byref(c)))
        self.q = w.q
        self.k_new, self.v_new = w.k_new, w.v_new
        self.tables = torch.from_numpy(w.block_tables).to(device)
        self.lens = torch.from_numpy(w.seq_lens).to(device)
        self.slots = torch.from_numpy(w.slot_mapping).to(device)
        self.pairs = torch.from_numpy(w.copy_pairs).to(device)
        self.npairs = int(w.copy_pairs.shape[0])
        self.cow = torch.from_numpy(cow_sources(w)).to(device)
        self.out = torch.empty_like(w.q)
        self.resident = dict(q=self.q, k_new=self.k_new, v_new=self.v_new, tables=self.tables,
                             lens=self.lens, slots=self.slots, pairs=self.pairs, cow=self.cow,
                             out=self.out)
        if mode not in ("cow", "fused", "two-call"):
            raise ValueError(f"unknown step mode {mode}")
        self.mode = mode
        # what a step reads from its inputs (the end-to-end run uploads these)
        self.input_keys = ["q", "k_new", "v_new", "tables", "lens"] + (
            ["cow"] if mode == "cow" else ["pairs"] + (["slots"] if mode == "two-call" else []))
        self.partition = int(partition)
        self.ws = pkv.make_workspace(self.N, self.Hq, H, D, w.max_blocks, B, self.partition,
                                     device=device)
        self.scale = ctypes.c_float(spec.scale)
        self.maxb = w.max_blocks
        self.fused = mode != "two-call"
        self.launches_per_step = ((1 if self.npairs and mode != "cow" else 0)
                                  + (2 if mode == "two-call" else 1) * self.L)

    def run(self, step_index, evl=None, bufs=None):
        """Launch one step; ``evl`` = per-layer (start, end) events around
        attention; ``bufs`` = the step's input/output tensors (default: the
        resident ones)."""
        lib = self.lib
        b = bufs if bufs is not None else self.resident
        _, cref = self.caches[step_index % len(self.caches)]
        rc = 0
        if self.npairs and self.mode != "cow":
            rc |= lib.pkv_block_copy(cref, b["pairs"].data_ptr(), self.npairs, self.sp)
        cow = b["cow"].data_ptr() if self.mode == "cow" else None
        for layer in range(self.L):
            if self.fused:                   # append (and copy-on-write) fused into attention
                if evl is not None:
                    evl[layer][0].record(self.stream)
                rc |= lib.pkv_append_paged_decode_attention(
                    cref, layer, b["k_new"][layer].data_ptr(), b["v_new"][layer].data_ptr(), cow,
                    b["q"][layer].data_ptr(), self.N, self.Hq, b["tables"].data_ptr(), self.maxb,
                    b["lens"].data_ptr(), self.scale, b["out"][layer].data_ptr(),
                    self.ws.data_ptr(), self.ws.numel(), self.partition, self.sp)
            else:
                rc |= lib.pkv_kv_append(cref, layer, b["k_new"][layer].data_ptr(),
                                        b["v_new"][layer].data_ptr(), b["slots"].data_ptr(),
                                        self.N, self.sp)
                if evl is not None:
                    evl[layer][0].record(self.stream)
                rc |= lib.pkv_paged_decode_attention(
                    cref, layer, b["q"][layer].data_ptr(), self.N, self.Hq, b["tables"].data_ptr(),
                    self.maxb, b["lens"].data_ptr(), self.scale, b["out"][layer].data_ptr(),
                    self.ws.data_ptr(), self.ws.numel(), self.partition, self.sp)
            if evl is not None:
                evl[layer][1].record(self.stream)
        if rc:
            raise RuntimeError(f"pagedkv call failed (status {rc})")


    def prepared(self, bufs=None):
        """The step as a list of library calls with every argument converted
        once (one list per pool replica); returns ``launch(step_index)``.
        Used where host time per step must stay well under device time."""
        lib = self.lib
        b = bufs if bufs is not None else self.resident
        ptr = lambda t: ctypes.c_void_p(t.data_ptr())
        cow = ptr(b["cow"]) if self.mode == "cow" else None
        per_replica = []
        for _, cref in self.caches:
            calls = []
            if self.npairs and self.mode != "cow":
                calls.append((lib.pkv_block_copy, (cref, ptr(b["pairs"]), self.npairs, self.sp)))
            for layer in range(self.L):
                if self.fused:
                    calls.append((lib.pkv_append_paged_decode_attention, (
                        cref, layer, ptr(b["k_new"][layer]), ptr(b["v_new"][layer]), cow,
                        ptr(b["q"][layer]), self.N, self.Hq, ptr(b["tables"]), self.maxb,
                        ptr(b["lens"]), self.scale, ptr(b["out"][layer]), ptr(self.ws),
                        self.ws.numel(), self.partition, self.sp)))
                else:
                    calls.append((lib.pkv_kv_append, (
                        cref, layer, ptr(b["k_new"][layer]), ptr(b["v_new"][layer]),
                        ptr(b["slots"]), self.N, self.sp)))
                    calls.append((lib.pkv_paged_decode_attention, (
                        cref, layer, ptr(b["q"][layer]), self.N, self.Hq, ptr(b["tables"]),
                        self.maxb, ptr(b["lens"]), self.scale, ptr(b["out"][layer]),
                        ptr(self.ws), self.ws.numel(), self.partition, self.sp)))
            per_replica.append(calls)

        def launch(step_index):
            rc = 0
            for fn, args in per_replica[step_index % len(per_replica)]:
                rc |= fn(*args)
            if rc:
                raise RuntimeError(f"pagedkv call failed (status {rc})")
        return launch


def packed_buffers(like, device, pin):
    """One contiguous byte buffer holding a tensor per entry of ``like`` (256-byte
    aligned views), so a step's inputs move in a single copy."""
    offs, total = {}, 0
    for k, t in like.items():
        offs[k] = total
        total += (t.numel() * t.element_size() + 255) // 256 * 256
    raw = torch.empty(total, dtype=torch.uint8, device=device, pin_memory=pin)
    views = {k: raw[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape)
             for (k, t), o in zip(like.items(), offs.values())}
    return raw, views


STEP_TEXT = {"cow": "per layer one launch: copy-on-write of shared tails, append of the new "
                    "token, attention",
             "fused": "block_copy, then per layer one fused append+attention launch",
             "two-call": "block_copy, then per layer kv_append and attention launches"}


L2_TEXT = ("inputs larger than L2: each step reads its own copy of the KV pools, rotating "
           "through copies that total at least 4x the L2 size")


def attention_tile_tokens(head_dim, block_size):
    """Tokens per pipeline stage of the attention kernel: a whole block at 32,
    32 at head_dim 64 with blocks of 8 or more, else 16."""
    if block_size >= 32:
        return block_size
    return 32 if head_dim == 64 and block_size >= 8 else 16


def rounded_partition(spec, B, requested):
    """The longest work range the attention call uses for ``requested``
    tokens (0 = no cap): rounded up to the kernel's tile.  Plain host
    arithmetic, so the reference arm can print it without the library."""
    if requested <= 0:
        return 0
    t = attention_tile_tokens(spec.head_dim, B)
    return -(-int(requested) // t) * t


def workload_config(key, spec, w, B, part, world, mode):
    """The ``config`` object both arms print for a workload."""
    return {"workload": key, "title": spec.title, "num_seqs": w.num_seqs,
            "num_layers": spec.num_layers, "q_heads": spec.num_q_heads,
            "kv_heads": spec.num_kv_heads, "head_dim": spec.head_dim, "block_size": B,
            "partition_tokens": rounded_partition(spec, B, part),
            "parallelism": f"dp{world} (independent batches, no collective)",
            "step": STEP_TEXT[mode], "l2": L2_TEXT}


def cow_sources(w):
    """Per sequence, the source block of this step's copy-on-write (-1 if
    none): the pair whose destination is the sequence's tail block."""
    src_of = {int(d): int(s) for s, d in w.copy_pairs}
    tails = w.block_tables[np.arange(w.num_seqs), (w.seq_lens.astype(np.int64) - 1) // w.block_size]
    return np.array([src_of.get(int(t), -1) for t in tails], np.int32)


def prestep_state(w):
    """The block manager's state before this step, from the step's outputs:
    lengths minus the new token, new tail blocks removed, copied tails mapped
    back to their sources, counts from the tables, free blocks in the
    workload's free-list order."""
    B = w.block_size
    lens = w.seq_lens.astype(np.int64) - 1
    tables = w.block_tables.copy()
    src_of = {int(d): int(s) for s, d in w.copy_pairs}
    NB = int(w.num_blocks)
    ref = np.zeros(NB, np.int64)
    for s in range(w.num_seqs):
        lb = int(lens[s]) // B
        if lens[s] % B == 0:
            tables[s, lb] = -1
        elif int(tables[s, lb]) in src_of:
            tables[s, lb] = src_of[int(tables[s, lb])]
        nblk = -(-int(lens[s]) // B)
        np.add.at(ref, tables[s, :nblk], 1)
    order = w.free_order if w.free_order is not None else np.arange(NB)
    free = np.array([b for b in order if ref[b] == 0], np.int32)
    ring = np.full(NB, -1, np.int32)
    ring[:len(free)] = free
    return dict(block_tables=tables.astype(np.int32), seq_lens=lens.astype(np.int32),
                refcount=ref.astype(np.int32), free_ring=ring,
                free_state=np.array([0, len(free)], np.int32))


def block_manager_timing(pkv, w, device, iters=100):
    """Mean device time of one block-manager step on this workload's pre-step
    state (restored, untimed, before every launch).  A 256 MB memset queued
    ahead of each timed launch keeps the GPU busy while the host enqueues, so
    the events see the kernel, not the host's call overhead."""
    from paged_kv_cache_378_b200._lib import PkvBlockState
    pristine = {k: torch.from_numpy(v).to(device) for k, v in prestep_state(w).items()}
    live = {k: v.clone() for k, v in pristine.items()}
    c = PkvBlockState(live["block_tables"].data_ptr(), live["seq_lens"].data_ptr(),
                      live["refcount"].data_ptr(), live["free_ring"].data_ptr(),
                      live["free_state"].data_ptr())
    N, maxb = live["block_tables"].shape
    order = None
    if w.batch_order is not None:        # the workload's writer order
        order = torch.from_numpy(np.ascontiguousarray(w.batch_order, dtype=np.int32)).to(device)
    slots = torch.empty(N, dtype=torch.int64, device=device)
    pairs = torch.empty((N, 2), dtype=torch.int32, device=device)
    npairs = torch.zeros(1, dtype=torch.int32, device=device)
    busy = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    lib = pkv.library()
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    args = (ctypes.byref(c), N, maxb, int(w.num_blocks), int(w.block_size),
            order.data_ptr() if order is not None else None, slots.data_ptr(), pairs.data_ptr(),
            npairs.data_ptr(), None, sp)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for i in range(iters + 5):
        for k in live:
            live[k].copy_(pristine[k])
        busy.zero_()
        if i >= 5:
            evs[i - 5][0].record(stream)
        if lib.pkv_block_manager_step(*args):
            raise SystemExit("block manager step refused its arguments")
        if i >= 5:
            evs[i - 5][1].record(stream)
    torch.cuda.synchronize(device)
    if pkv.get_device_status(reset=True):
        raise SystemExit("device status raised by the block manager step")
    return sum(a.elapsed_time(b) for a, b in evs) / iters * 1e3


def block_manager_chained_timing(pkv, w, gs, device, steps=40, chunks=10):
    """Device time the block-manager step adds when it runs between chained
    attention launches (the device-only decode loop), against the launches
    alone: median over chunks of `steps` steps.  The step works on its own
    copy of the pre-step state (tables with spare columns so no sequence
    outgrows them), restored before every chunk; the attention launches read
    the workload's own inputs, so their work is the same in both."""
    from paged_kv_cache_378_b200._lib import PkvBlockState
    st = prestep_state(w)
    bt = st["block_tables"]
    st["block_tables"] = np.concatenate([bt, np.full((bt.shape[0], 16), -1, bt.dtype)], axis=1)
    pristine = {k: torch.from_numpy(np.ascontiguousarray(v)).to(device) for k, v in st.items()}
    live = {k: v.clone() for k, v in pristine.items()}
    c = PkvBlockState(live["block_tables"].data_ptr(), live["seq_lens"].data_ptr(),
                      live["refcount"].data_ptr(), live["free_ring"].data_ptr(),
                      live["free_state"].data_ptr())
    N, maxb = live["block_tables"].shape
    order = None
    if w.batch_order is not None:
        order = torch.from_numpy(np.ascontiguousarray(w.batch_order, dtype=np.int32)).to(device)
    slots = torch.empty(N, dtype=torch.int64, device=device)
    pairs = torch.empty((N, 2), dtype=torch.int32, device=device)
    npairs = torch.zeros(1, dtype=torch.int32, device=device)
    cow = torch.empty(N, dtype=torch.int32, device=device)
    lib = pkv.library()
    args = (ctypes.byref(c), N, maxb, int(w.num_blocks), int(w.block_size),
            ctypes.c_void_p(order.data_ptr()) if order is not None else None,
            ctypes.c_void_p(slots.data_ptr()), ctypes.c_void_p(pairs.data_ptr()),
            ctypes.c_void_p(npairs.data_ptr()), ctypes.c_void_p(cow.data_ptr()), gs.sp)
    launch = gs.prepared()

    def chunk(with_step):
        for k in live:
            live[k].copy_(pristine[k])
        torch.cuda._sleep(SPIN_CYCLES)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(gs.stream)
        for i in range(steps):
            launch(i)
            if with_step and lib.pkv_block_manager_step(*args):
                raise SystemExit("block manager step refused its arguments")
        e1.record(gs.stream)
        torch.cuda.synchronize(device)
        return e0.elapsed_time(e1) / steps * 1e3

    for _ in range(2):
        chunk(True)
        chunk(False)
    alone = float(np.median([chunk(False) for _ in range(chunks)]))
    both = float(np.median([chunk(True) for _ in range(chunks)]))
    if pkv.get_device_status(reset=True):
        raise SystemExit("device status raised by the chained block manager steps")
    return alone, both


def prefix_hash_timing(pkv, w, device, iters=50):
    """Mean device time of hashing every full block of the batch (token ids
    drawn per physical slot, so shared prompts share blocks); a memset queued
    ahead of each launch hides the host's call overhead from the events."""
    from workload import token_ids
    tok = torch.from_numpy(token_ids(w)).to(device)
    lens = torch.from_numpy(w.seq_lens).to(device)
    N, T = tok.shape
    mb = T // w.block_size
    out = torch.zeros((N, mb), dtype=torch.int64, device=device)
    busy = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    lib = pkv.library()
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for i in range(iters + 3):
        busy.zero_()
        if i >= 3:
            evs[i - 3][0].record(stream)
        if lib.pkv_prefix_block_hashes(tok.data_ptr(), T, lens.data_ptr(), None, None, None, N,
                                       w.block_size, out.data_ptr(), mb, sp):
            raise SystemExit("prefix hash refused its arguments")
        if i >= 3:
            evs[i - 3][1].record(stream)
    torch.cuda.synchronize(device)
    if pkv.get_device_status(reset=True):
        raise SystemExit("device status raised by the prefix hash")
    us = sum(a.elapsed_time(b) for a, b in evs) / iters * 1e3
    blocks = int(sum(int(n) // w.block_size for n in w.seq_lens))
    return {"us": us, "full_blocks": blocks, "blocks_per_s": blocks / (us * 1e-6),
            "token_bytes_gbs": blocks * w.block_size * 4 / (us * 1e-6) / 1e9,
            "what": "FNV-1a 64 chain hash of every full block (parent hash, block tokens, "
                    "extra key), one warp per sequence"}


def prefix_hash_decode_timing(pkv, w, device, iters=50):
    """Mean device time of the per-step (decode) form of the prefix hash: each
    sequence hashes only its newest full block, resuming the chain from the
    stored hash of the block before it (``first_block``/``parent_hashes``).
    Every sequence is given one block to hash (the last full one), the most a
    decode step can ask for."""
    from workload import token_ids
    tok = torch.from_numpy(token_ids(w)).to(device)
    lens_np = w.seq_lens.astype(np.int64)
    full = lens_np // w.block_size
    first = np.maximum(full - 1, 0).astype(np.int32)
    lens = torch.from_numpy(w.seq_lens).to(device)
    first_d = torch.from_numpy(first).to(device)
    N, T = tok.shape
    mb = T // w.block_size
    parents = torch.zeros(N, dtype=torch.int64, device=device)   # stored hashes (values do not matter for time)
    out = torch.zeros((N, mb), dtype=torch.int64, device=device)
    busy = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    lib = pkv.library()
    stream = torch.cuda.current_stream(device)
    sp = ctypes.c_void_p(stream.cuda_stream)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(iters)]
    for i in range(iters + 3):
        busy.zero_()
        if i >= 3:
            evs[i - 3][0].record(stream)
        if lib.pkv_prefix_block_hashes(tok.data_ptr(), T, lens.data_ptr(), None, first_d.data_ptr(),
                                       parents.data_ptr(), N, w.block_size, out.data_ptr(), mb, sp):
            raise SystemExit("prefix hash (decode form) refused its arguments")
        if i >= 3:
            evs[i - 3][1].record(stream)
    torch.cuda.synchronize(device)
    if pkv.get_device_status(reset=True):
        raise SystemExit("device status raised by the prefix hash (decode form)")
    us = sum(a.elapsed_time(b) for a, b in evs) / iters * 1e3
    blocks = int((full > 0).sum())
    return {"us": us, "blocks": blocks, "blocks_per_s": blocks / (us * 1e-6),
            "what": "decode form: one newly full block per sequence, chain resumed from the "
                    "stored parent hash"}


def swap_timing(pkv, w, device, blocks=1024, iters=10):
    """Block swap out to / back in from a pinned host pool: GB/s each way, and
    a plain pinned cudaMemcpy of the same bytes each way for reference."""
    L, NB, H, B, D = w.k_pool.shape
    m = min(blocks, NB)
    hk = torch.empty((L, m, H, B, D), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    rng = np.random.default_rng(0)
    dev_ids = rng.choice(NB, m, replace=False).astype(np.int32)
    out_pairs = torch.from_numpy(np.stack([dev_ids, np.arange(m, dtype=np.int32)], 1)).to(device)
    in_pairs = torch.from_numpy(np.stack([np.arange(m, dtype=np.int32), dev_ids], 1)).to(device)
    nbytes = 2 * hk.numel() * hk.element_size()
    stream = torch.cuda.current_stream(device)
    ref_h = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    ref_d = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def timed(fn):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(iters):
            fn()
        e1.record(stream)
        e1.synchronize()
        return e0.elapsed_time(e1) / iters * 1e-3

    t_out = timed(lambda: pkv.swap_blocks(out_pairs, w.k_pool, w.v_pool, hk, hv, pkv.SWAP_OUT))
    t_in = timed(lambda: pkv.swap_blocks(in_pairs, w.k_pool, w.v_pool, hk, hv, pkv.SWAP_IN))
    t_h2d = timed(lambda: ref_d.copy_(ref_h, non_blocking=True))
    t_d2h = timed(lambda: ref_h.copy_(ref_d, non_blocking=True))
    if pkv.get_device_status(reset=True):
        raise SystemExit("device status raised by the block swap")
    return {"blocks": m, "bytes_each_way": nbytes,
            "out_gbs": nbytes / t_out / 1e9, "in_gbs": nbytes / t_in / 1e9,
            "memcpy_d2h_gbs": nbytes / t_d2h / 1e9, "memcpy_h2d_gbs": nbytes / t_h2d / 1e9,
            "what": "swap of randomly chosen device blocks (all layers, K and V) to a pinned "
                    "host pool and back, one launch each way; reference: one pinned memcpy of "
                    "the same bytes"}


def e2e_run(pkv, w, gs, steps, device):
    """The same step through the C ABI from host buffers.  Every step uploads
    its inputs (what the step reads: q, k_new, v_new, block tables, lengths,
    and the copy sources, or the copy pairs and slot mapping; one packed
    pinned buffer, one copy) and reads its attention output
    back to pinned host memory.  Three buffer sets rotate, so later steps'
    uploads and earlier steps' downloads run on copy streams while step i
    computes."""
    # host threads and pinned buffers on the GPU's NUMA node: copies then
    # cross no socket link
    local = gpu_local_cpus(pci_bus_id(device.index if device.index is not None else 0))
    if local:
        os.sched_setaffinity(0, local)
    every = dict(q=w.q.cpu(), k_new=w.k_new.cpu(), v_new=w.v_new.cpu(),
                 tables=torch.from_numpy(w.block_tables), lens=torch.from_numpy(w.seq_lens),
                 slots=torch.from_numpy(w.slot_mapping), pairs=torch.from_numpy(w.copy_pairs),
                 cow=torch.from_numpy(cow_sources(w)))
    host_src = {k: every[k] for k in gs.input_keys}
    h_raw, h_views = packed_buffers(host_src, "cpu", True)
    for k, t in host_src.items():
        h_views[k].copy_(t)
    SETS = 3                                    # buffer sets in flight
    dev = [packed_buffers(host_src, device, False) for _ in range(SETS)]
    outs = [torch.empty_like(gs.out) for _ in range(SETS)]
    out_host = [torch.empty(gs.out.shape, dtype=gs.out.dtype).pin_memory() for _ in range(SETS)]
    h2d = h_raw.numel()
    d2h = out_host[0].numel() * out_host[0].element_size()
    comp = gs.stream
    up = torch.cuda.Stream(device)
    down = torch.cuda.Stream(device)
    ev = lambda: torch.cuda.Event()
    uploaded = [ev() for _ in range(SETS)]
    computed = [ev() for _ in range(SETS)]
    downloaded = [ev() for _ in range(SETS)]
    for e in computed + downloaded:
        e.record(comp)
    launches = [gs.prepared(dict(dev[k][1], out=outs[k])) for k in range(SETS)]

    def one(i):
        k = i % SETS
        up.wait_event(computed[k])                  # the step that last used this set is done
        with torch.cuda.stream(up):
            dev[k][0].copy_(h_raw, non_blocking=True)
        uploaded[k].record(up)
        comp.wait_event(uploaded[k])
        comp.wait_event(downloaded[k])              # that step's output has left
        launches[k](i)
        computed[k].record(comp)
        down.wait_event(computed[k])
        with torch.cuda.stream(down):
            out_host[k].copy_(outs[k], non_blocking=True)
        downloaded[k].record(down)

    for i in range(4):
        one(i)
    torch.cuda.synchronize(device)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    up.wait_event(e0)
    for i in range(steps):
        one(i)
    comp.wait_event(downloaded[(steps - 1) % SETS])  # the last output is on the host
    e1.record(comp)
    e1.synchronize()
    torch.cuda.synchronize(device)
    # same inputs as the resident run and a deterministic schedule: same bits
    if not torch.equal(out_host[(steps - 1) % SETS], gs.out.cpu()):
        raise SystemExit("end-to-end output differs from the resident run's")
    return e0.elapsed_time(e1) / steps, h2d, d2h, (len(local) if local else None)


# ---------------------------------------------------------------------------
# the oracle on the host (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------

def _u16(t):
    return t.contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def oracle_full_step(oa, w, host):
    """The oracle's whole step on every sequence: copies, append, attention."""
    L = w.spec.num_layers
    kp, vp = oa.block_copy(host["k"], host["v"], w.copy_pairs)
    for layer in range(L):
        k2, v2 = oa.kv_append(kp[layer], vp[layer], host["k_new"][layer], host["v_new"][layer],
                              w.slot_mapping, w.block_size)
        oa.paged_decode_attention(host["q"][layer], k2, v2, w.block_tables, w.seq_lens,
                                  w.block_size, w.spec.scale)


def cpu_threads_used():
    try:
        from threadpoolctl import threadpool_info
        return max([1] + [int(i.get("num_threads", 1)) for i in threadpool_info()])
    except Exception:
        return 1


def limit_blas_threads():
    try:
        from threadpoolctl import threadpool_limits
        return threadpool_limits(1)
    except Exception:
        return None


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def host_workload(key, block_size, seed):
    w = make_workload(key, block_size=block_size, seed=seed, device="cpu", poison=False)
    host = dict(k=_u16(w.k_pool), v=_u16(w.v_pool), q=_u16(w.q), k_new=_u16(w.k_new),
                v_new=_u16(w.v_new))
    return w, host


def cpu_baseline_single(w, host, unique_bytes, min_seconds=10.0):
    """The oracle's whole step, one thread (BLAS pinned to 1), repeated for
    about ``min_seconds``."""
    from oracle import attention as oa
    lim = limit_blas_threads()
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle_full_step(oa, w, host)
        n += 1
        if time.perf_counter() - t0 >= min_seconds:
            break
    dt = (time.perf_counter() - t0) / n
    cores = cpu_threads_used() if lim is None else 1
    return {"value": unique_bytes * w.spec.num_layers / dt / 1e9, "unit": UNIT, "cores": cores,
            "kind": "oracle",
            "sample": f"the whole step of this workload (all {w.num_seqs} sequences: block_copy, "
                      f"kv_append, attention, {w.spec.num_layers} layer(s)), repeated {n}x, "
                      f"{dt:.2f} s per step, numpy fp64, 1 thread"}


# -- the oracle over every host core: a process pool over sequences --------------
# Workers are started with ``spawn`` (never forked from a process that has
# touched the GPU) and read the step's pools from shared memory.

_POOL_STATE = {}


def _pool_worker_init(shm_specs, meta):
    from multiprocessing import shared_memory
    limit_blas_threads()
    arrays, handles = {}, []
    for k, (name, shape, dtype) in shm_specs.items():
        shm = shared_memory.SharedMemory(name=name)
        handles.append(shm)
        arrays[k] = np.ndarray(shape, dtype=np.dtype(dtype), buffer=shm.buf)
    _POOL_STATE.update(arrays)
    _POOL_STATE["_handles"] = handles
    _POOL_STATE["meta"] = meta


def _pool_worker_attention(idx):
    """The oracle's attention for sequences ``idx``, every layer."""
    from oracle import attention as oa
    P = _POOL_STATE
    m = P["meta"]
    idx = np.asarray(idx, dtype=np.int64)
    for layer in range(m["L"]):
        oa.paged_decode_attention(P["q"][layer][idx], P["k2"][layer], P["v2"][layer],
                                  P["tables"][idx], P["lens"][idx], m["B"], m["scale"])
    return len(idx)


def cpu_baseline_all_cores(w, host, unique_bytes, min_seconds=10.0):
    """The oracle's whole step with its attention spread over a ``spawn``
    process pool, one worker per core of ``os.sched_getaffinity(0)``: the
    parent runs the oracle's block_copy and kv_append, the workers the
    oracle's attention on balanced groups of sequences.  Returns None where
    a pool cannot be started."""
    import multiprocessing as mp
    from multiprocessing import shared_memory
    from oracle import attention as oa
    cores = len(os.sched_getaffinity(0))
    L = w.spec.num_layers
    kp, vp = oa.block_copy(host["k"], host["v"], w.copy_pairs)
    k2 = np.empty_like(kp)
    v2 = np.empty_like(vp)
    for layer in range(L):
        k2[layer], v2[layer] = oa.kv_append(kp[layer], vp[layer], host["k_new"][layer],
                                            host["v_new"][layer], w.slot_mapping, w.block_size)
    arrays = {"q": host["q"], "k2": k2, "v2": v2, "tables": w.block_tables, "lens": w.seq_lens}
    shms, specs = [], {}
    try:
        for k, a in arrays.items():
            shm = shared_memory.SharedMemory(create=True, size=max(1, a.nbytes))
            shms.append(shm)
            np.ndarray(a.shape, dtype=a.dtype, buffer=shm.buf)[...] = a
            specs[k] = (shm.name, a.shape, a.dtype.str)
        # groups of sequences of about equal KV bytes, 4 per worker
        lens = w.seq_lens.astype(np.int64)
        ngroups = max(1, min(w.num_seqs, 4 * cores))
        groups = [[] for _ in range(ngroups)]
        load = np.zeros(ngroups)
        for s in np.argsort(-lens, kind="stable").tolist():
            g = int(np.argmin(load))
            groups[g].append(s)
            load[g] += lens[s] + 1
        groups = [g for g in groups if g]
        meta = {"L": L, "B": w.block_size, "scale": w.spec.scale}
        ctx = mp.get_context("spawn")
        with ctx.Pool(cores, initializer=_pool_worker_init, initargs=(specs, meta)) as pool:
            pool.map(_pool_worker_attention, [[0]] * cores)          # start and warm every worker
            lim = limit_blas_threads()
            n = 0
            t0 = time.perf_counter()
            while True:
                kq, vq = oa.block_copy(host["k"], host["v"], w.copy_pairs)
                for layer in range(L):
                    oa.kv_append(kq[layer], vq[layer], host["k_new"][layer], host["v_new"][layer],
                                 w.slot_mapping, w.block_size)
                pool.map(_pool_worker_attention, groups, chunksize=1)
                n += 1
                if time.perf_counter() - t0 >= min_seconds:
                    break
            dt = (time.perf_counter() - t0) / n
            del lim
    except (OSError, RuntimeError) as e:
        return {"unavailable": f"{type(e).__name__}: {e}"}
    finally:
        for shm in shms:
            shm.close()
            shm.unlink()
    return {"value": unique_bytes * L / dt / 1e9, "unit": UNIT, "cores": cores,
            "kind": "oracle", "cpu_model": cpu_model(),
            "sample": f"the whole step of this workload (all {w.num_seqs} sequences, "
                      f"{L} layer(s)): block_copy and kv_append in the parent, attention over "
                      f"{len(groups)} balanced groups of sequences on a spawn pool of {cores} "
                      f"worker processes (one per core of sched_getaffinity, BLAS 1 thread each); "
                      f"repeated {n}x, {dt:.2f} s per step, numpy fp64"}


def cpu_baseline(key, block_size, seed, unique_bytes, min_seconds=10.0):
    """Both oracle timings on the host: one thread, and every core."""
    w, host = host_workload(key, block_size, seed)
    one = cpu_baseline_single(w, host, unique_bytes, min_seconds)
    every = cpu_baseline_all_cores(w, host, unique_bytes, min_seconds)
    if every is None or "unavailable" in every:
        one["all_cores"] = every
        return one
    every["single_thread"] = one
    return every


def run_reference(args):
    """--impl reference: the oracle timed as it stands on the host cores.
    Touches neither the GPU nor this repository's library."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from oracle import attention as oa
    spec = get_spec(args.workload)
    B = args.block_size or spec.block_size
    lim = limit_blas_threads()
    w, host = host_workload(args.workload, B, spec.seed)
    part = spec.partition_tokens if args.partition < 0 else args.partition
    ref_config = workload_config(args.workload, spec, w, B, part,
                                 int(os.environ.get("WORLD_SIZE", "1")), args.step)
    kp, vp = oa.block_copy(host["k"], host["v"], w.copy_pairs)
    k2, v2 = oa.kv_append(kp[0], vp[0], host["k_new"][0], host["v_new"][0], w.slot_mapping,
                          w.block_size)
    per_seq_bytes = w.seq_lens.astype(np.int64) * 2 * spec.num_kv_heads * spec.head_dim * 2
    # calibrate: seconds per KV byte of the oracle's attention
    cal = list(range(0, w.num_seqs, max(1, w.num_seqs // 8)))
    t = time.perf_counter()
    oa.paged_decode_attention(host["q"][0][cal], k2, v2, w.block_tables[cal], w.seq_lens[cal],
                              w.block_size, spec.scale)
    s_per_byte = (time.perf_counter() - t) / max(1, int(per_seq_bytes[cal].sum()))
    budget = 120.0 / (args.steps + args.warmup)
    target = budget / s_per_byte
    m = int(np.clip(np.searchsorted(np.cumsum(per_seq_bytes), target), 1, w.num_seqs))

    def step(i):
        idx = [(i * m + j) % w.num_seqs for j in range(m)]
        oa.paged_decode_attention(host["q"][0][idx], k2, v2, w.block_tables[idx], w.seq_lens[idx],
                                  w.block_size, spec.scale)
        return int(per_seq_bytes[idx].sum())

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    tot = 0
    for i in range(args.steps):
        tot += step(args.warmup + i)
    dt = time.perf_counter() - t0
    val = tot / dt / 1e9
    cores = 1 if lim is not None else cpu_threads_used()
    sample = (f"attention of {m} of {w.num_seqs} sequences per step (round robin), layer 0, after "
              f"the oracle's block_copy and kv_append of the step; numpy fp64")
    line = {"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT,
            "n_gpus": int(os.environ.get("WORLD_SIZE", args.gpus)), "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": ref_config,
            "cpu_baseline": {"value": val, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# measurement of a step made of attention launches only (copy-on-write folded in)
# ---------------------------------------------------------------------------

def algorithmic_bytes(w, spec, B, gs, unique_bytes):
    """Algorithmic bytes of one attention launch (one layer): unique K/V, q
    and out, tables and lengths, and with the fused append the new tokens'
    K/V read and stored, and with the folded copy-on-write the copied tail
    blocks written."""
    q_out = 2 * w.num_seqs * spec.num_q_heads * spec.head_dim * 2
    meta = w.block_tables.nbytes + w.seq_lens.nbytes
    append = 2 * (2 * w.num_seqs * spec.num_kv_heads * spec.head_dim * 2) if gs.fused else 0
    cow = (gs.npairs * spec.num_kv_heads * B * spec.head_dim * 2 * 2) if gs.mode == "cow" else 0
    return {"unique_kv": unique_bytes, "q_out": q_out, "tables_lengths": meta,
            "append": append, "copy_on_write": cow,
            "total": unique_bytes + q_out + meta + append + cow}


def region_ms(gs, steps, first=0):
    """Device time of ``steps`` chained steps (CUDA events on the launching stream)."""
    fast = gs.prepared()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(gs.stream)
    for i in range(steps):
        fast(first + i)
    e1.record(gs.stream)
    e1.synchronize()
    return e0.elapsed_time(e1)


def launch_stats(gs, steps, first=0):
    """Per-launch attention times from a separate, untimed pass with events
    around every launch (each launch then runs alone: no overlap with the
    one before it), in microseconds."""
    L = gs.L
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(L)] for _ in range(steps)]
    for i in range(steps):
        gs.run(first + i, evs[i])
    torch.cuda.synchronize(gs.device)
    us = sorted(a.elapsed_time(b) * 1e3 for row in evs for a, b in row)

    def q(p):
        return us[min(len(us) - 1, int(round(p * (len(us) - 1))))]
    return {"launches": len(us), "median_us": q(0.5), "p10_us": q(0.1), "p90_us": q(0.9),
            "min_us": us[0], "max_us": us[-1],
            "what": "each attention launch bracketed by CUDA events in a separate pass "
                    "(launches then do not overlap their neighbours)"}


def peak_fractions(gbs, peak):
    return {"pct_of_8tbs": 100.0 * gbs / NOMINAL_HBM_GBS, "pct_of_measured": 100.0 * gbs / peak}


def measure_config(pkv, key, B, part, device, sampler, peak, peak_kind, min_region_s=0.3):
    """One workload at one block size through the default step (one launch per
    layer: copy-on-write, append, attention): value, roofline, clocks and
    per-launch statistics, for the ``per_config`` part of the line."""
    spec = get_spec(key)
    w = make_workload(key, block_size=B, seed=spec.seed, device=device, poison=False)
    unique = w.unique_kv_bytes_read()
    pool_bytes = 2 * w.k_pool.numel() * w.k_pool.element_size()
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nrep = max(1, min(16, math.ceil(4 * l2 / pool_bytes)))
    replicas = [(w.k_pool, w.v_pool)] + [(w.k_pool.clone(), w.v_pool.clone())
                                         for _ in range(nrep - 1)]
    gs = GpuStep(pkv, w, replicas, part, device, mode="cow")
    pkv.get_device_status(reset=True)
    for i in range(5):
        gs.run(i)
    est = region_ms(gs, 3, 5) / 3
    steps = max(20, int(math.ceil(min_region_s * 1e3 / max(est, 1e-3))))
    torch.cuda.synchronize(device)
    wall0 = time.time()
    torch.cuda._sleep(SPIN_CYCLES)
    ms = region_ms(gs, steps, 8)
    wall1 = time.time()
    stats = launch_stats(gs, max(8, min(200, int(math.ceil(200 / spec.num_layers)))), 8 + steps)
    status = pkv.get_device_status(reset=True)
    if status:
        raise SystemExit(f"device status {status:#x} raised while measuring {key} B={B}")
    ms_step = ms / steps
    value = unique * spec.num_layers / (ms_step * 1e-3) / 1e9
    alg = algorithmic_bytes(w, spec, B, gs, unique)
    launch_us = ms_step * 1e3 / spec.num_layers
    achieved = alg["total"] / (launch_us * 1e-6) / 1e9
    out = {"workload": key, "block_size": B,
           "partition_tokens": rounded_partition(spec, B, part),
           "num_seqs": w.num_seqs, "num_layers": spec.num_layers,
           "value": value, "unit": UNIT, "steps": steps, "ms_per_step": ms_step,
           "decode_tokens_per_s_per_layer": w.num_seqs * spec.num_layers / (ms_step * 1e-3),
           "kv_bytes_per_step": {"unique": unique * spec.num_layers,
                                 "logical": w.kv_bytes_read() * spec.num_layers},
           **peak_fractions(value, peak),
           "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                        "frac": achieved / peak, "kernel": "paged_attention_kernel",
                        "alg_bytes_per_launch": alg, "avg_launch_us": launch_us,
                        "peak_source": f"{peak_kind} hbm_gbs"},
           "launch_stats": stats,
           "clocks": sampler.summary(wall0 - 0.05, wall1 + 0.05),
           "l2": f"{nrep} rotating copies of the KV pools, {nrep * pool_bytes / 1e9:.2f} GB vs "
                 f"{l2 / 1e6:.0f} MB L2"}
    del gs, replicas, w
    torch.cuda.empty_cache()
    return out


PER_CONFIG = [("llama1b_layer", 16, -1), ("long_context", 16, -1), ("long_context", 16, 0),
              ("full_step", 8, -1), ("full_step", 16, -1), ("full_step", 32, -1)]


# ---------------------------------------------------------------------------
# main (our arm)
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--block-size", type=int, default=0)
    ap.add_argument("--partition", type=int, default=-1, help="-1: the workload's, 0: library default")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the other workloads' lines (per_config)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the block-manager, swap and prefix-hash timings")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--soak-seconds", type=float, default=1.5)
    ap.add_argument("--step", choices=["cow", "fused", "two-call"], default="cow",
                    help="cow (default): one launch per layer doing copy-on-write, append and "
                         "attention; fused: block_copy, then append+attention per layer; "
                         "two-call: block_copy, then kv_append and attention per layer")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    spec = get_spec(args.workload)
    B = args.block_size or spec.block_size
    part = spec.partition_tokens if args.partition < 0 else args.partition
    seed = rank_seed(spec.seed, rank)

    w_meta = make_workload(args.workload, block_size=B, seed=seed, values=False)
    unique_bytes = w_meta.unique_kv_bytes_read()
    logical_bytes = w_meta.kv_bytes_read()

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=device)

    import paged_kv_cache_378_b200 as pkv

    sampler = ClockSampler(pci_bus_id(local)).start()

    w = make_workload(args.workload, block_size=B, seed=seed, device=device, poison=False)
    rounded = pkv.partition_tokens(w.num_seqs, spec.num_kv_heads, spec.head_dim, w.max_blocks, B,
                                   part)
    if rounded != rounded_partition(spec, B, part):
        raise SystemExit("partition rounding differs from the library's")
    pool_bytes = 2 * w.k_pool.numel() * w.k_pool.element_size()
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    nrep = max(1, min(16, math.ceil(4 * l2 / pool_bytes)))
    replicas = [(w.k_pool, w.v_pool)] + [(w.k_pool.clone(), w.v_pool.clone()) for _ in range(nrep - 1)]
    gs = GpuStep(pkv, w, replicas, part, device, mode=args.step)
    pkv.get_device_status(reset=True)

    # warm-up
    for i in range(args.warmup):
        gs.run(i)
    torch.cuda.synchronize(device)
    if pkv.get_device_status(reset=True):
        raise SystemExit("device status raised during warm-up")

    # When the attention kernel is the only kernel of the step (copy-on-write
    # folded in), every launch in the timed region is that kernel and its
    # average duration is the timed region over the launches.  Otherwise
    # attention is bracketed by events on every EVENT_EVERY-th step only: an
    # event between two kernels ends their programmatic overlap, so the other
    # steps run chained as a user's stream would.
    only_attention = gs.mode == "cow"
    ev_steps = [] if only_attention else list(range(0, args.steps, EVENT_EVERY))
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(len(ev_steps) * spec.num_layers)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize(device)
    wall0 = time.time()
    # A spin kernel ahead of the region keeps the GPU busy while the host
    # enqueues the steps, so the events time the device, not the host's
    # first enqueue latency (a short region would otherwise include it).
    # NVTX ranges mark the phases for a profiler's timeline (one push and
    # pop per phase, none per launch)
    torch.cuda.nvtx.range_push("timed steps")
    torch.cuda._sleep(SPIN_CYCLES)
    t_start.record(gs.stream)
    nl = spec.num_layers
    fast = gs.prepared()
    for i in range(args.steps):
        j = i // EVENT_EVERY
        if not only_attention and i % EVENT_EVERY == 0:
            gs.run(i, evs[j * nl:(j + 1) * nl])
        else:
            fast(i)
    t_end.record(gs.stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(device)
    wall1 = time.time()
    if dist is not None:
        dist.barrier()
    ms = t_start.elapsed_time(t_end)
    soak_until = wall1
    if wall1 - wall0 < args.soak_seconds:      # keep the GPU busy so the clock sampler sees load
        i = args.steps
        while time.time() - wall0 < args.soak_seconds:
            for _ in range(50):
                gs.run(i)
                i += 1
            torch.cuda.synchronize(device)
        soak_until = time.time()
    clocks = sampler.summary(wall0 - 0.05, soak_until + 0.05)
    clocks["window"] = "timed region" if soak_until == wall1 else "timed region + untimed soak"
    status = pkv.get_device_status(reset=True)
    if status:
        raise SystemExit(f"device status {status:#x} raised in the timed region")

    if only_attention:
        attn_ms = [ms / (args.steps * spec.num_layers)] * (args.steps * spec.num_layers)
        sampling = "every launch in the timed region is this kernel: timed region / launches"
    else:
        attn_ms = [a.elapsed_time(b) for a, b in evs]
        sampling = f"attention bracketed on every {EVENT_EVERY}th timed step"
    attn_avg_ms = sum(attn_ms) / len(attn_ms)
    # per-launch distribution from a separate untimed pass (every launch alone)
    with torch.cuda.nvtx.range("per-launch statistics"):
        stats = launch_stats(gs, max(50, min(500, args.steps)), args.steps + 10**6)

    # totals over ranks: device time is the max, work is the sum
    ms_max, bytes_total, seqs_total = combine_over_ranks(
        dist, ms, unique_bytes * spec.num_layers, w.num_seqs, device)
    ms_per_step = ms_max / args.steps
    value = bytes_total / (ms_per_step * 1e-3) / 1e9

    e2e = None
    if not args.no_e2e:
        with torch.cuda.nvtx.range("end to end"):
            e_ms, h2d, d2h, ncpu = e2e_run(pkv, w, gs, args.e2e_steps, device)
        e_ms = combine_over_ranks(dist, e_ms, 0, 0, device)[0]
        e2e = {"value": bytes_total / (e_ms * 1e-3) / 1e9, "unit": UNIT,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "ms_per_step": e_ms, "steps": args.e2e_steps,
               "pipeline": "three buffer sets: uploads and downloads of neighbouring steps on copy streams while step i computes",
               "host_cpus": f"{ncpu} GPU-local CPUs" if ncpu else "affinity unchanged"}

    extras = {}
    if not args.no_extras:
        torch.cuda.nvtx.range_push("rows beyond attention")
        bm_us = block_manager_timing(pkv, w, device) if w.num_seqs <= 4096 else None
        bm_chain = (block_manager_chained_timing(pkv, w, gs, device)
                    if bm_us is not None and spec.num_layers == 1 else None)
        extras["swap"] = swap_timing(pkv, w, device)
        extras["prefix_hash"] = prefix_hash_timing(pkv, w, device)
        extras["prefix_hash_decode"] = prefix_hash_decode_timing(pkv, w, device)
        extras["block_manager"] = None if bm_us is None else {
            "us_per_step": bm_us, "num_seqs": w.num_seqs,
            "what": "device block-manager step (slot mapping, copy-on-write decisions, block "
                    "allocation) timed alone on this step's pre-step state, restored between launches"}
        if bm_chain is not None:
            extras["block_manager"].update({
                "chained_attention_us": bm_chain[0], "chained_with_step_us": bm_chain[1],
                "added_between_chained_launches_us": bm_chain[1] - bm_chain[0],
                "chained_what": "attention launches chained back to back, with and without the "
                                "step between them (it reads and decides before its wait on the "
                                "previous launch, so only its writes and the next launch's start "
                                "are added)"})
        torch.cuda.nvtx.range_pop()

    peak, peak_kind = load_peak()
    alg = algorithmic_bytes(w, spec, B, gs, unique_bytes)
    achieved = alg["total"] / (attn_avg_ms * 1e-3) / 1e9
    traffic = load_traffic(args.workload, B, gs.mode, gs.partition)
    launches_per_step = gs.launches_per_step
    del gs, replicas, w
    torch.cuda.empty_cache()

    # the other workloads, each through the same step (rank 0 at N = 1 only;
    # ranks of a multi-GPU run take the same collective steps without these)
    per_config = None
    if world == 1 and not args.no_per_config:
        per_config = []
        for key, bs, p in PER_CONFIG:
            sp = get_spec(key)
            with torch.cuda.nvtx.range(f"config {key} B={bs} partition={p}"):
                per_config.append(measure_config(pkv, key, bs, sp.partition_tokens if p < 0 else p,
                                                 device, sampler, peak, peak_kind))
    sampler.stop()

    # the oracle on the host cores last: a spawned pool, so starting it after
    # this process used the GPU is safe (rank 0 at N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(args.workload, B, seed, unique_bytes)

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(args.workload, spec, w_meta, B, part, world, args.step),
        "l2_detail": f"{nrep} rotating copies of the KV pools, {nrep * pool_bytes / 1e9:.2f} GB vs "
                     f"{l2 / 1e6:.0f} MB L2",
        "pct_hbm_peak": 100.0 * value / peak,
        **peak_fractions(value, peak),
        # one token per sequence per layer: N x L tokens cross a layer per step
        "decode_tokens_per_s_per_layer": seqs_total * spec.num_layers / (ms_per_step * 1e-3),
        "kv_bytes_per_step": {"unique": unique_bytes * spec.num_layers,
                              "logical": logical_bytes * spec.num_layers},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "kernel": "paged_attention_kernel", "alg_bytes_per_launch": alg["total"],
                     "alg_bytes_parts": alg,
                     "avg_launch_us": attn_avg_ms * 1e3, "peak_source": f"{peak_kind} hbm_gbs",
                     "timed_launches": len(attn_ms),
                     "event_sampling": sampling},
        "launch_stats": stats,
        "cpu_baseline": cpu,
        "e2e": e2e,
        **extras,
        "per_config": per_config,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())

"""The N > 1 host path on CPU: two gloo ranks, each with its own independent
batch (weak scaling, no data-path collective); the timing reduction takes the
max device time and sums the work."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from workload import make_workload, rank_seed


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = make_workload("continuous_batch", seed=rank_seed(3, rank), values=False)
        ms = 1.5 + rank                     # rank 1 is the slow one
        res = bench.combine_over_ranks(dist, ms, w.unique_kv_bytes_read(), w.num_seqs,
                                       torch.device("cpu"))
        out[rank] = (res, w.unique_kv_bytes_read(), w.seq_lens.sum())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timing_and_work():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn",
                       join=True)
    (ms0, b0, s0), own0, _ = out[0]
    (ms1, b1, s1), own1, _ = out[1]
    assert ms0 == ms1 == 2.5                     # max over ranks
    assert b0 == b1 == own0 + own1               # whole-job bytes
    assert s0 == s1 == 512
    assert own0 != own1                          # independent batches


def test_rank_batches_are_independent_and_reproducible():
    a0 = make_workload("llama1b_layer", seed=rank_seed(2, 0), values=False)
    a1 = make_workload("llama1b_layer", seed=rank_seed(2, 1), values=False)
    b1 = make_workload("llama1b_layer", seed=rank_seed(2, 1), values=False)
    assert rank_seed(2, 0) == 2
    assert not np.array_equal(a0.seq_lens, a1.seq_lens)
    assert np.array_equal(a1.seq_lens, b1.seq_lens)
    assert np.array_equal(a1.block_tables, b1.block_tables)


def test_single_process_combine_is_identity():
    assert bench.combine_over_ranks(None, 3.0, 10, 4, None) == (3.0, 10.0, 4.0)


def test_reference_arm_on_non_zero_rank_does_nothing(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), {"workload": "tiny", "block_size": 0, "steps": 3, "warmup": 3, "gpus": 2})
    assert bench.run_reference(args) == 0
    assert capsys.readouterr().out == ""


def test_reference_arm_prints_one_line(monkeypatch, capsys):
    import json
    monkeypatch.setenv("RANK", "0")
    args = type("A", (), {"workload": "tiny", "block_size": 0, "steps": 3, "warmup": 3, "gpus": 1,
                          "partition": -1, "step": "cow"})
    assert bench.run_reference(args) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    # the same config object the GPU arm prints for this workload
    assert line["config"]["workload"] == "tiny" and line["config"]["num_seqs"] == 4
    assert line["config"]["step"] == bench.STEP_TEXT["cow"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["cpu_baseline"]["kind"] == "oracle"

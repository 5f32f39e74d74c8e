"""The N > 1 bookkeeping of bench.py on 2 gloo ranks (CPU): every rank draws its own
batch (or, split by heads, its own range of one job's heads), the job time is the
slowest rank's, and the job throughput counts every rank's work. The data path itself
has no collective (heads and batches are independent)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import workloads as W


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _head_worker(rank, world, port, H, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        gathered = [None] * world
        dist.all_gather_object(gathered, bench.shard_heads(H, world, rank))
        out[rank] = gathered
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("H", [24, 3, 1])
def test_head_split_covers_every_head_once_on_gloo_ranks(H):
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_head_worker, args=(world, _free_port(), H, out), nprocs=world, join=True,
                       start_method="spawn")
    ranges = out[0]
    assert ranges == out[1]                    # every rank sees the same partition
    owned = [h for a, b in ranges for h in range(a, b)]
    assert owned == list(range(H))             # contiguous, each head exactly once


@pytest.mark.parametrize("world", [1, 2, 3, 5, 8, 30])
def test_head_partition_sizes(world):
    H = 24
    ranges = [bench.shard_heads(H, world, r) for r in range(world)]
    assert [h for a, b in ranges for h in range(a, b)] == list(range(H))
    sizes = [b - a for a, b in ranges]
    assert max(sizes) - min(sizes) <= 1


def test_head_split_inputs_are_the_one_gpu_job_heads():
    """A rank that owns heads [a, b) draws exactly those heads of the one-GPU job, so the
    ranks' outputs together are the one-GPU output."""
    wl = W.get("tiny").with_(H=5)
    full = W.make_inputs(wl)
    for world in (2, 3):
        for r in range(world):
            a, b = bench.shard_heads(wl.H, world, r)
            part = W.make_inputs(wl, heads=list(range(a, b)))
            for x, y in zip(part, full):
                assert np.array_equal(x, y[:, a:b])


def test_gpus_flag_starts_the_ranks(monkeypatch):
    """--gpus N without a torchrun environment starts N ranks through torchrun."""
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    seen = {}

    def fake_call(cmd):
        seen["cmd"] = cmd
        return 0
    monkeypatch.setattr(bench.subprocess, "call", fake_call)
    assert bench.main(["--gpus", "4", "--steps", "3", "--warmup", "3", "--shard", "heads"]) == 0
    cmd = " ".join(seen["cmd"])
    assert "torch.distributed.run" in cmd and "--nproc-per-node=4" in cmd
    assert "--master-addr 127.0.0.1" in cmd and cmd.rstrip().endswith("--shard heads")


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = W.get("tiny").with_(H=2)
        q, _, _ = W.make_inputs(wl, batch_offset=bench.rank_batch_offset(wl, rank))
        gathered = [None] * world
        dist.all_gather_object(gathered, q.tobytes())
        mx = bench.max_over_ranks(10.0 + rank, dist, torch.device("cpu"))
        out[rank] = (mx, gathered[0] != gathered[1], bench._dist())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for rank in range(world):
        mx, distinct, (ws, r, local) = out[rank]
        assert mx == 11.0                      # slowest rank
        assert distinct                        # ranks hold different batches
        assert (ws, r, local) == (world, rank, rank)


def test_job_throughput_counts_every_rank():
    assert bench.job_throughput(1e12, 4, 10.0) == pytest.approx(400.0)


def test_single_rank_defaults(monkeypatch):
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench._dist() == (1, 0, 0)
    assert bench.max_over_ranks(3.5, None, torch.device("cpu")) == 3.5


def test_rank_batches_are_independent_draws():
    wl = W.get("tiny")
    a = W.make_inputs(wl, batch_offset=0)[0]
    b = W.make_inputs(wl, batch_offset=1)[0]
    two = W.make_inputs(wl.with_(B=2))[0]
    assert not np.array_equal(a, b)
    assert np.array_equal(two[1:], b)          # rank 1's batch == batch 1 of a 2-batch job

"""The bench's multi-rank host logic on CPU: two gloo ranks (no GPU).

Every rank runs its own batch (replicas, weak scaling); the reported time is
the max over ranks and the units (bytes, tokens) are summed.  The reference
arm prints from rank 0 only; the other ranks exit 0 without work.
"""
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
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        times, units = bench.reduce_over_ranks([1.0 + rank, 10.0 * (rank + 1)],
                                               [100.0 * (rank + 1), 4096.0, 7.0], "cpu")
        w = bench.replica_workload(W.get("M4096-zipf1.1"), rank)
        idx = W.make_routing(w)
        gathered = [None] * world
        dist.all_gather_object(gathered, idx[:64].tolist())
        q.put((rank, times, units, gathered))
    finally:
        dist.destroy_process_group()


def test_two_rank_reduction_and_replica_batches():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, times, units, gathered in res:
        assert times == [2.0, 20.0]                       # max over ranks
        assert units == [300.0, 8192.0, 14.0]             # sums over ranks
        assert gathered[0] != gathered[1]                 # each replica its own batch
        assert np.array(gathered[0]).shape == (64, 8)


def test_single_process_reduction_is_identity():
    assert bench.reduce_over_ranks([3.0], [5.0, 6.0], "cpu") == ([3.0], [5.0, 6.0])


def test_reference_arm_only_on_rank0(monkeypatch, capsys):
    monkeypatch.setenv("RANK", "1")
    args = bench.main.__globals__["argparse"].Namespace(steps=1, warmup=3, gpus=2)
    assert bench.run_reference(args, W.get("M4096-zipf1.1")) == 0
    assert capsys.readouterr().out == ""


def test_algorithmic_bytes_formulas():
    w = W.get("M4096-zipf1.1")
    b = bench.algorithmic_bytes(w, 32768, 32768)
    M, N, k = 4096, 7168, 8
    assert b["dispatch"] == 2 * M * N + 32768 * N * 2 + 4 * M * k
    assert b["combine"] == 2 * 32768 * N + 2 * M * N + 8 * M * k
    w5 = W.get("prefill-M65536-mix-dedup-fp8")
    b5 = bench.algorithmic_bytes(w5, 524288, 334500)
    assert b5["dispatch"] == 2 * 65536 * N + 334500 * N + 4 * 334500 * 56 + 4 * 65536 * 8

"""The benchmark's multi-GPU plumbing on CPU with two gloo ranks: each rank takes
a disjoint slice of one token stream, its seeded inputs are exactly that slice
of the single-process stream, the job's step time is the slowest rank's, and
the reference arm runs on rank 0 only. The data path has no collective (rows
are independent), so nothing else crosses ranks."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, M, K, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import torch.distributed as dist

    import bench
    import synth
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        row0, rows = bench.shard_rows(rank, world, M)
        x = synth.activation_host(0, synth.tensor_ids()["x"], np.arange(row0, row0 + rows), K)
        slowest = bench.max_over_ranks(10.0 + rank)  # rank r "took" 10 + r ms
        q.put((rank, row0, rows, x.sum(dtype=np.int64), slowest))
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_rows_and_time_by_the_slowest():
    world, M, K = 2, 24, 256
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, M, K, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    import synth
    full = synth.activation_host(0, synth.tensor_ids()["x"], np.arange(world * M), K)
    covered = []
    for rank, row0, rows, checksum, slowest in got:
        assert rows == M
        covered.extend(range(row0, row0 + rows))
        assert checksum == full[row0:row0 + rows].sum(dtype=np.int64)
        assert slowest == 10.0 + (world - 1)
    assert sorted(covered) == list(range(world * M))


def test_job_throughput_counts_all_ranks():
    import bench
    assert bench.job_tops(1e12, 1, 1.0) == pytest.approx(1000.0)
    assert bench.job_tops(1e12, 4, 2.0) == pytest.approx(2000.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    import bench
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = type("A", (), dict(workload="tiny", M=None, F=None, steps=1, warmup=0))()
    assert bench.run_reference(args) == 0  # returns at once, prints nothing

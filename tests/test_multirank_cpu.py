"""The multi-GPU host logic of the bench, run as two gloo ranks on the CPU.

The layer shards over tokens with no exchange, so `bench.py --gpus N` runs N
weak-scaled replicas; the only cross-rank step is the max-over-ranks timing
reduction and the whole-job throughput built from it.  These tests run that
logic in two processes on 127.0.0.1 without a GPU.
"""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    w, r, local = bench.dist_setup(world)
    assert (w, r, local) == (world, rank, rank)
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        # rank r took (r + 1) * 10 ms for 3 steps of 1e12 operations
        local_ms = (rank + 1) * 10.0
        tops, total_ms = bench.weak_scaling_throughput(1e12, 3, local_ms, world, torch.device("cpu"))
        out[rank] = (tops, total_ms, bench.max_over_ranks(float(rank), world, torch.device("cpu")))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_weak_scaling_reduction_two_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert set(res) == {0, 1}
    for rank in range(world):
        tops, total_ms, mx = res[rank]
        assert total_ms == pytest.approx(20.0)           # the slower rank
        assert mx == 1.0
        # 2 ranks x 3 steps x 1e12 ops in 20 ms = 300 TOP/s
        assert tops == pytest.approx(2 * 3 * 1e12 / 0.020 / 1e12)


def test_single_rank_needs_no_process_group():
    import bench
    tops, total_ms = bench.weak_scaling_throughput(2e12, 4, 8.0, 1, torch.device("cpu"))
    assert total_ms == 8.0 and tops == pytest.approx(4 * 2e12 / 0.008 / 1e12)


def test_world_size_must_match_gpus(monkeypatch):
    import bench
    monkeypatch.setenv("WORLD_SIZE", "4")
    with pytest.raises(SystemExit):
        bench.dist_setup(2)


def test_issue_loop_measurement_failure_keeps_the_bench_line():
    """The tensor-core rate is context for the roofline: if measuring it fails,
    the bench reports None instead of losing its JSON line."""
    import bench

    class Failing:
        @staticmethod
        def measure_int8_mma_rate(iters):
            raise RuntimeError("no device")

    class Working:
        @staticmethod
        def measure_int8_mma_rate(iters):
            assert iters == 32768
            return 4321.0

    assert bench.issue_loop_tops(Failing()) is None
    assert bench.issue_loop_tops(Working()) == 4321.0

"""The multi-rank plumbing of bench.py ("replicas only": no data-path
collective) on CPU with gloo, world size 2: every rank agrees on the slowest
rank's time, the job value counts every rank's tokens, the reference arm
does its work on rank 0 only, and `--gpus N` without a launcher spawns N
ranks of its own with a working process group."""
import datetime
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import torch
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
        v = bench.job_value(world, 4096, 100, ms)

        class A:
            workload, steps, warmup, gpus = "tiny_fp32", 1, 0, world
        ref = bench.run_reference(A, rank, world) if rank != 0 else "skipped"
        dist.barrier()
        q.put((rank, ms, v, ref))
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_value():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert [o[1] for o in out] == [15.0, 15.0]  # both ranks see the max
    assert out[0][2] == pytest.approx(2 * 4096 * 100 / 0.015)
    assert out[1][3] is None  # the reference arm does no work off rank 0


def test_single_process_value_is_plain_throughput():
    sys.path.insert(0, ROOT)
    import bench
    import torch
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.job_value(1, 4096, 10, 20.0) == pytest.approx(4096 * 10 / 0.02)


def test_reference_arm_runs_the_oracle_on_rank0():
    sys.path.insert(0, ROOT)
    import bench

    class A:
        workload, steps, warmup, gpus = "tiny_fp32", 2, 1, 1
    line = bench.run_reference(A, 0, 1)
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def _spawned_probe(q, rank, world):
    import torch
    import bench
    ms = bench.max_over_ranks(10.0 + 5.0 * rank, torch.device("cpu"))
    q.put((rank, world, int(os.environ["LOCAL_RANK"]), ms))


def test_bench_spawns_its_own_ranks():
    import functools
    import multiprocessing

    sys.path.insert(0, ROOT)
    import bench
    q = multiprocessing.get_context("spawn").Queue()
    codes = bench.launch_local_ranks(2, functools.partial(_spawned_probe, q), "gloo",
                                     timeout_s=60)
    assert codes == [0, 0]
    out = sorted(q.get(timeout=30) for _ in range(2))
    assert [o[:3] for o in out] == [(0, 2, 0), (1, 2, 1)]
    assert [o[3] for o in out] == [15.0, 15.0]

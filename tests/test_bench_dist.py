"""The multi-rank logic of bench.py on the CPU: two ``gloo`` ranks in spawned
processes reduce their timings to the maximum over ranks, and the whole-job
value counts every rank's work against that slowest time (weak scaling)."""

import datetime
import importlib.util
import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import torch.distributed as dist

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        # rank r took (1 + r) ms for the step and (10 - r) ms end to end
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank], world, "cpu")
        value = bench.job_tflops(world, 1e12, 4, got[0])
        dist.barrier()
        q.put((rank, got, value))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_value_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in procs:
            rank, got, value = q.get(timeout=120)
            results[rank] = (got, value)
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
    assert all(p.exitcode == 0 for p in procs)
    for rank in (0, 1):
        got, value = results[rank]
        assert got == [2.0, 10.0]  # the slowest rank's time, on every rank
        # 2 ranks x 1 TFLOP per step x 4 steps in 2 ms
        assert value == pytest.approx(2 * 1e12 * 4 / 2e-3 / 1e12)


def test_single_rank_is_the_identity():
    bench = _bench()
    assert bench.max_over_ranks([3.5, 1.25], 1, "cpu") == [3.5, 1.25]
    assert bench.job_tflops(1, 2e12, 10, 20.0) == pytest.approx(1000.0)

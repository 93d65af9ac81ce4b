"""Multi-rank host logic of bench.py on CPU: two gloo ranks (no GPU).

Each rank of a replicas-only run times its own work; the reported numbers are
the maximum over ranks of the timings and the whole job's units over that
time.  The GPU path runs the same helpers over NCCL.
"""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _bench()
        # rank r's timings: prefill 10 + r ms, decode 100 - 5 r ms, total 7 r
        got = bench.max_over_ranks([10.0 + rank, 100.0 - 5 * rank, 7.0 * rank], world, "cpu")
        rate = bench.whole_job_rate(128, world, got[1])
        dist.barrier()
        out[rank] = (got, rate)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_rate_two_gloo_ranks():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        got, rate = out[r]
        assert got == [11.0, 100.0, 7.0]           # element-wise max over the ranks
        assert rate == pytest.approx(2 * 128 / 0.1)  # all ranks' units / slowest time


def test_single_rank_is_identity():
    bench = _bench()
    assert bench.max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
    assert bench.whole_job_rate(256, 1, 500.0) == pytest.approx(512.0)

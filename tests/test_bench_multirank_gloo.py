"""bench.py's multi-rank aggregation, run as world_size-2 gloo ranks on CPU: the step time is
the slowest rank's, the whole-job rate counts every rank's work over that time, and a step
that needs every rank (the end-to-end leg) runs only if all ranks can run it."""

import importlib.util
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _load_bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench = _load_bench()
        elapsed = [100.0, 130.0][rank]                 # rank 1 is the slow one
        slowest = bench.max_over_ranks(elapsed, "cpu")
        agree_yes = bench.all_ranks(True, "cpu")
        agree_no = bench.all_ranks(rank == 0, "cpu")   # rank 1 cannot run it
        rate = bench.whole_job_rate(1e12, world, 5, slowest)
        out_q.put((rank, slowest, agree_yes, agree_no, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=240) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, slowest, yes, no, rate in res:
        assert slowest == 130.0                        # both ranks see the slowest rank's time
        assert yes is True and no is False
        assert abs(rate - 1e12 * 2 * 5 / 0.130) < 1e3  # all ranks' work over the slowest time


def test_single_process_needs_no_group():
    bench = _load_bench()
    assert bench.max_over_ranks(7.0, "cpu") == 7.0
    assert bench.all_ranks(False, "cpu") is False
    assert bench.whole_job_rate(10.0, 1, 2, 1000.0) == 20.0

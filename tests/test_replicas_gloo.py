"""The N > 1 bench path ("replicas only": one independent replica per GPU)
on CPU: two gloo ranks on 127.0.0.1 reduce their per-rank timings to the
maximum, as bench.py does on GPUs with NCCL, and the whole-job throughput is
computed from the slowest rank."""
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
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench = _bench()
        # rank r: step 10 + r ms, outer 5 - r ms -> max is (10 + world - 1, 5)
        out = bench.max_over_ranks(dist, [10.0 + rank, 5.0 - rank], "cpu")
        dist.barrier()
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == {0: [11.0, 5.0], 1: [11.0, 5.0]}


def test_single_process_and_job_value():
    bench = _bench()
    assert bench.max_over_ranks(None, [3, 4.5], "cpu") == [3.0, 4.5]
    # two replicas of 1 TFLOP each, slowest rank 2 ms per step -> 1000 TFLOP/s
    assert bench.job_tflops(2, 1e12, 2.0) == pytest.approx(1000.0)
    assert bench.job_tflops(1, 1e12, 2.0) == pytest.approx(500.0)

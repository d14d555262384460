"""The multi-rank logic of bench.py on CPU: two gloo ranks run the same reductions the
GPU ranks run over NCCL. The path does not shard ("replicas only"): every rank times its
own replica, the job's rate is the units of all ranks over the slowest rank's time."""

import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        mx = bench.max_over_ranks(1.5 + rank, world)          # 1.5, 2.5
        sm = bench.sum_over_ranks(10.0 * (rank + 1), world)   # 10 + 20
        # rank 0 processed 100 units in 2 s, rank 1 300 units in 4 s: 400 units / 4 s
        rate = bench.job_throughput(100.0 if rank == 0 else 300.0, 2.0 if rank == 0 else 4.0, world)
        bench.barrier(world)
        q.put((rank, mx, sm, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_like_the_gpu_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=240)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    res = sorted(q.get() for _ in range(2))
    for rank, mx, sm, rate in res:
        assert mx == pytest.approx(2.5)
        assert sm == pytest.approx(30.0)
        assert rate == pytest.approx(100.0)


def test_single_rank_is_the_identity():
    sys.path.insert(0, ROOT)
    import importlib.util
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    assert bench.max_over_ranks(3.0, 1) == 3.0
    assert bench.sum_over_ranks(3.0, 1) == 3.0
    assert bench.job_throughput(300.0, 2.0, 1) == pytest.approx(150.0)
    assert torch.distributed.is_available()

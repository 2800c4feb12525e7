"""Host logic of bench.py's N > 1 path, on world-size-2 gloo ranks (CPU only).

With several GPUs the bench runs independent replicas; the only cross-rank
steps are the barrier and the max-over-ranks time, exercised here.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dist.barrier()
        ms = [7.0, 11.5][rank]
        worst = bench.max_over_ranks(ms, torch.device("cpu"))
        q.put((rank, worst, bench.job_tflops(world, 1e12, worst)))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    out = sorted(q.get(timeout=10) for _ in range(2))
    for rank, worst, tflops in out:
        assert worst == 11.5
        assert tflops == pytest.approx(2 * 1e12 / 11.5e-3 / 1e12)


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.25, torch.device("cpu")) == 3.25

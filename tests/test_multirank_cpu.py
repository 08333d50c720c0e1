"""Multi-rank plumbing of bench.py on CPU (world size 2, gloo): the job time is the max over
ranks, the value is the weak-scaling total, and only rank 0 of the reference arm reports.
The path itself has no data-path collective (each rank runs its own IndexShare group)."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, ws, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(ws),
                      LOCAL_RANK=str(rank))
    import datetime
    import torch.distributed as dist
    import bench
    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        t = bench.max_over_ranks(10.0 + 5.0 * rank, ws)          # rank 1 is the slow one
        v = bench.job_throughput(32768, 4, ws, t)
        out.put((rank, t, v))
        # the reference arm: ranks other than 0 return without work or output
        class A:
            workload, seq_len, steps, warmup, ref_seconds = "tiny_prefill", 64, 1, 0, 0.5
        if rank != 0:
            assert bench.run_reference(A, ws, rank) is None
    finally:
        dist.destroy_process_group()


def test_two_rank_timing_and_weak_scaling():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, t, v in res:
        assert t == 15.0                                  # max over ranks
        assert v == pytest.approx(32768 * 2 * 4 / 0.015)  # both ranks' tokens over the slowest time

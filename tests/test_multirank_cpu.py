"""The multi-rank plumbing of bench.py on CPU: two gloo ranks agree on the
max-over-ranks time and on the whole-job (weak scaling) throughput."""

import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, out):
    import datetime

    import torch.distributed as dist

    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=ws, timeout=datetime.timedelta(seconds=60))
    try:
        bench.barrier(ws)
        ms = 10.0 * (rank + 1)                  # rank 1 is the slowest
        out[rank] = (bench.max_over_ranks(ms, ws), bench.job_throughput(1000.0, ws, ms))
        bench.barrier(ws)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_agree():
    ws = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        out = m.dict()
        mp.start_processes(_worker, args=(ws, _free_port(), out), nprocs=ws, join=True,
                           start_method="spawn")
        res = dict(out)
    assert res[0] == res[1]
    mx, thr = res[0]
    assert mx == 20.0
    assert thr == pytest.approx(1000.0 * 2 / 0.020)

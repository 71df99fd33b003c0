"""The multi-GPU bench path on the host: two ranks over gloo on CPU.

`bench.py --gpus N` runs N replicas (each rank its own batch; the path has no
exchange step) and reports the job's time as the slowest rank's.  The reduction
it uses is checked here with two processes and the gloo backend, so no GPU is
needed.
"""
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


def _rank_main(rank, world, port, value, out):
    import datetime

    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        out.put((rank, bench.max_over_ranks(value, world, torch.device("cpu"))))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_slowest_rank_time_over_gloo():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    values = [3.25, 7.5]                   # per-rank step times: the job's is 7.5
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, values[r], out)) for r in range(2)]
    for p in procs:
        p.start()
    got = {}
    try:
        for _ in range(2):
            r, v = out.get(timeout=120)
            got[r] = v
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.terminate()
    assert got == {0: 7.5, 1: 7.5}
    assert all(p.exitcode == 0 for p in procs)


def test_single_rank_time_is_its_own():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(4.5, 1, None) == 4.5

"""The benchmark's multi-rank bookkeeping on CPU with the gloo backend, world size 2:
every rank gets the slowest rank's time, and the whole-job rate counts every rank's
units (weak scaling: per-rank work is fixed)."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    local_ms = [12.5, 20.0][rank]
    got = bench.max_over_ranks(local_ms, torch.device("cpu"))
    rate = bench.weak_scaling_rate(1e12, world, got)
    q.put((rank, got, rate))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_weak_scaling_with_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in range(2)]
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for rank, got, rate in res:
        assert got == 20.0
        assert abs(rate - 2e12 / 20e-3) < 1e-3 * rate


def test_single_process_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, torch.device("cpu")) == 3.5
    assert bench.weak_scaling_rate(10.0, 1, 1000.0) == 10.0

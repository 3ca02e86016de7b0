"""The benchmark's multi-rank host logic on CPU: two `gloo` ranks (one
process per rank, as torchrun starts them) meet at the barrier, take the max
of their times, and aggregate the bytes of all ranks over that time.  The
product path itself is replicas only (no collective on the data path)."""
import importlib.util
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world,
                                         timeout=datetime.timedelta(seconds=30))
    try:
        b = _bench()
        b.barrier(world)
        t = 1.5 if rank == 0 else 2.5            # rank 1 is the slower one
        t_max = b.max_over_ranks(world, t)
        rate = b.aggregate_rate(1e9, 10, t_max, world)
        b.barrier(world)
        out.put((rank, t_max, rate))
    finally:
        torch.distributed.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time_and_all_bytes():
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(out.get(timeout=5) for _ in range(2))
    for rank, t_max, rate in res:
        assert t_max == 2.5
        assert rate == pytest.approx(1e9 * 10 * 2 / 2.5 / 1e9)   # 8 GB/s over both ranks


def test_single_rank_needs_no_process_group():
    b = _bench()
    assert b.max_over_ranks(1, 3.0) == 3.0
    b.barrier(1)
    assert b.aggregate_rate(30322688, 100, 0.001, 1) == pytest.approx(30322688 * 100 / 0.001 / 1e9)

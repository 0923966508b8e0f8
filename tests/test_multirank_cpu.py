"""The bench's multi-rank host logic on CPU, world size 2 over gloo: device
times are combined as the max over ranks, the whole-job value counts every
rank's bytes over the slowest rank's time, the barrier joins both ranks, and
the reference arm (the oracle on the host cores) runs on rank 0 only.  No GPU
and no NCCL: the bench runs independent replicas, so these are its only
cross-rank steps."""
import importlib.util
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("rq_bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        b = _bench()
        b.barrier(world)
        ms = [3.0, 5.0][rank]                       # this rank's device time
        m = b.max_over_ranks(ms, world)
        value = b.job_gbs(world, 1e9, 10, m)       # 1 GB per rank and step, 10 steps
        # the reference arm returns at once on every rank but 0
        ref = b.reference_arm(None, None, rank, world) if rank != 0 else "rank0"
        out.put((rank, m, value, ref))
        b.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_ranks_over_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        rank, m, value, ref = out.get(timeout=120)
        res[rank] = (m, value, ref)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank in range(world):
        m, value, _ = res[rank]
        assert m == 5.0                             # the slower rank's time, on every rank
        assert value == pytest.approx(2 * 1e9 * 10 / 5e-3 / 1e9)
    assert res[1][2] is None                        # no work on rank 1


def test_single_rank_is_identity():
    b = _bench()
    assert b.max_over_ranks(7.5, 1) == 7.5
    assert b.job_gbs(1, 2e9, 4, 8.0) == pytest.approx(2e9 * 4 / 8e-3 / 1e9)

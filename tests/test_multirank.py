"""The N > 1 plumbing of bench.py on CPU with gloo, world size 2: process-group
set-up, barrier, max-over-ranks timing, and rank-0-only reporting of the
reference arm."""
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    import torch.distributed as dist
    r, w, _ = bench.dist_setup("reference")
    assert (r, w) == (rank, world)
    bench.barrier(w)
    # each rank reports a different step time; every rank must see the slowest
    m = bench.max_over_ranks(1.5 + r, w)
    # the reference arm runs on rank 0 only: other ranks return without work
    class A:
        steps, warmup, seed = 1, 0, 0
    if r != 0:
        assert bench.run_reference(A, r, w) is None
    out[rank] = m
    dist.destroy_process_group()


def test_two_rank_gloo_max_over_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(out) == {0: 2.5, 1: 2.5}

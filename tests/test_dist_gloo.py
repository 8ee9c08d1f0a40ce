"""Weak-scaling plumbing on two CPU ranks (gloo): sharding and max-over-ranks timing."""

import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    from hybrid_sliding_window_sink_b200 import dist as D
    try:
        w, r = D.init("gloo", timeout_s=60)
        assert (w, r) == (world, rank)
        # every unit lands on exactly one rank, blocks differ by at most one unit
        for n in (0, 1, 7, 16384, 16385):
            lo, hi = D.shard_range(n, r, w)
            tot = D.sum_over_ranks(hi - lo)
            assert tot == n
        # the job time is the slowest rank's
        t = 10.0 + 5.0 * r
        assert D.max_over_ranks(t) == 10.0 + 5.0 * (world - 1)
        D.barrier()
        q.put((rank, "ok"))
    except Exception as e:  # report to the parent
        q.put((rank, repr(e)))
    finally:
        D.finalize()


def test_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == {0: "ok", 1: "ok"}


def test_shard_range_single_process():
    from hybrid_sliding_window_sink_b200 import dist as D
    assert D.shard_range(10, 0, 1) == (0, 10)
    blocks = [D.shard_range(10, r, 3) for r in range(3)]
    assert blocks == [(0, 4), (4, 7), (7, 10)]

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


def _decode_shard_worker(rank, world, port, q):
    """Each rank computes its block of (sequence, KV head) units of a ring decode, a linear
    decode and a sparse decode with the oracle; the gathered blocks must equal the unsharded
    oracle bit for bit (the units share nothing)."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    import numpy as np
    import torch.distributed as dist
    from hybrid_sliding_window_sink_b200 import dist as D, workloads as wl
    from oracle import ref
    try:
        D.init("gloo", timeout_s=60)
        B, hq, hkv, cap = 5, 16, 4, 300
        G = hq // hkv
        lengths = [300, 1, 129, 77, 250]
        d = wl.decode_inputs(B, hq, hkv, cap, lengths, seed=90)
        qf, kc, vc, sk = (wl.to_f64(d[k]) for k in ("q", "k_cache", "v_cache", "sink"))
        lens_sp = [300, 100, 129, 85, 250]
        sel = wl.sorted_unique_indices(B, hkv, 20, [x - 64 for x in lens_sp], seed=90).numpy()
        calls = {
            "ring": (lambda q_, k_, v_, L_, s_, sl: ref.decode(q_, k_[:, :128], v_[:, :128], "ring", L_, s_), lengths),
            "linear": (lambda q_, k_, v_, L_, s_, sl: ref.decode(q_, k_, v_, "linear", L_, s_), lengths),
            "sparse": (lambda q_, k_, v_, L_, s_, sl: ref.sparse_decode(q_, k_, v_, L_, 64, sl, s_), lens_sp),
        }
        for name, (fn, lens) in calls.items():
            mine = {}
            for b, g in D.unit_shard(B, hkv, rank, world):
                hs = slice(g * G, (g + 1) * G)
                mine[(b, g)] = fn(qf[b:b + 1, hs], kc[b:b + 1, :, g:g + 1], vc[b:b + 1, :, g:g + 1], [lens[b]],
                                  sk[hs], sel[b:b + 1, g:g + 1])
            parts = [None] * world
            dist.all_gather_object(parts, mine)
            o = np.full((B, hq, 128), np.nan)
            l = np.full((B, hq), np.nan)
            for part in parts:
                for (b, g), (ob, lb) in part.items():
                    o[b, g * G:(g + 1) * G] = ob[0]
                    l[b, g * G:(g + 1) * G] = lb[0]
            o_full, l_full = fn(qf, kc, vc, lens, sk, sel)
            assert np.array_equal(o, o_full) and np.array_equal(l, l_full), name
        q.put((rank, "ok"))
    except Exception as e:  # report to the parent
        q.put((rank, repr(e)))
    finally:
        D.finalize()


@pytest.mark.parametrize("world", [2, 3])
def test_decode_partition_is_exact(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_decode_shard_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert res == {r: "ok" for r in range(world)}


def test_unit_shard_covers_every_unit_once():
    from hybrid_sliding_window_sink_b200 import dist as D
    for B, hkv, world in ((64, 8, 8), (64, 4, 3), (5, 4, 2), (1, 1, 4)):
        units = [u for r in range(world) for u in D.unit_shard(B, hkv, r, world)]
        assert units == [(b, g) for b in range(B) for g in range(hkv)]


def test_shard_range_single_process():
    from hybrid_sliding_window_sink_b200 import dist as D
    assert D.shard_range(10, 0, 1) == (0, 10)
    blocks = [D.shard_range(10, r, 3) for r in range(3)]
    assert blocks == [(0, 4), (4, 7), (7, 10)]

"""Timing of the float64 oracle on the host's cores: the benchmark's CPU baseline.

TEST INFRASTRUCTURE, NOT PRODUCT CODE. Only the ``cpu_baseline`` and ``--impl reference``
legs of ``bench.py`` run this module, as a separate process that never touches a GPU:

    python -m oracle.baseline [--budget SECONDS] [--only NAME] [--steps K --warmup W]

It prints one JSON object. The oracle functions run as they stand (``oracle/ref.py``); this
module only builds inputs of the benchmark workloads' shapes and distributions (N(0,1)
values drawn in float64; the oracle's time does not depend on the values) and spreads
independent rows over a pool of worker processes, one per core, each with one BLAS thread.
Throughput counts the algorithmic work of the rows computed over the wall time of the pool.

Workloads (the benchmark's configurations):
  tiny_prefill   SWA prefill n=1024, 8 Q / 1 KV, W=128          every row (full)
  swa_prefill    SWA prefill n=32768, 64 Q / 8 KV, W=128        row sample, extrapolated
  ga_prefill     GA prefill n=32768 causal, 64 Q / 4 KV         row sample, extrapolated
  swa_decode     one SWA decode layer, B=64, ring 128, 64/8     every row (full)
  ga_decode      one GA decode layer, B=64, L ~ U[4096, 131072], 64/4
                                                                sequence sample, extrapolated
  sparse_decode  B=8, L=262144, 64/4, recent 128 + 1024         every row (full)
Extrapolation is by the work count (score pairs for prefill, cached key rows for decode):
the oracle spends the same time per pair whichever row it belongs to.
"""

from __future__ import annotations

import argparse
import json
import os
import sys
import time

# one BLAS thread per worker process; set before numpy loads
for _v in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ[_v] = "1"

import math  # noqa: E402
import multiprocessing as mp  # noqa: E402

import numpy as np  # noqa: E402

from oracle import ref  # noqa: E402

DQK, DV = 192, 128
FLOP_PER_PAIR = 2.0 * (DQK + DV)
BYTES_PER_KEY = (DQK + DV) * 2          # one bf16 K row and V row per (token, KV head)

# Inputs are built in the parent before the pool forks, and read (never written) by the
# workers, so every worker shares the parent's pages.
_DATA: dict = {}


def _rng(seed):
    return np.random.default_rng(seed)


def _swa_pairs(n, window):
    if window <= 0 or window >= n:
        return n * (n + 1) // 2
    return n * window - window * (window - 1) // 2


# ----------------------------------------------------------------------------- inputs
def _build(names, seed=2000):
    r = _rng(seed)
    if "tiny_prefill" in names:
        n, hq, hkv = 1024, 8, 1
        _DATA["tiny_prefill"] = dict(q=r.standard_normal((1, n, hq, DQK)), k=r.standard_normal((1, n, hkv, DQK)),
                                     v=r.standard_normal((1, n, hkv, DV)), sink=r.standard_normal(hq))
    for name, hq, hkv, window, theta in (("swa_prefill", 64, 8, 128, 1e4), ("ga_prefill", 64, 4, 0, 1e7)):
        if name not in names:
            continue
        n = 32768
        # K rotated once by the oracle's rope (a whole-layer call rotates K once as well);
        # the sampled query rows are rotated per row inside the timed region
        k = r.standard_normal((n, hkv, DQK))
        t0 = time.perf_counter()
        kr = ref.rope(k, np.arange(n, dtype=np.float64), theta, 64)
        t_rope = time.perf_counter() - t0
        _DATA[name] = dict(kr=kr, v=r.standard_normal((n, hkv, DV)), sink=r.standard_normal(hq), n=n,
                           hq=hq, hkv=hkv, window=window, theta=theta, t_rope=t_rope,
                           qseed=seed + (1 if window else 2))
    if "swa_decode" in names:
        B, hq, hkv, cap = 64, 64, 8, 128
        _DATA["swa_decode"] = dict(q=r.standard_normal((B, hq, DQK)), kc=r.standard_normal((B, cap, hkv, DQK)),
                                   vc=r.standard_normal((B, cap, hkv, DV)), sink=r.standard_normal(hq),
                                   lengths=r.integers(4096, 131072 + 1, size=B))
    if "ga_decode" in names:
        # one shared cache of 131072 tokens for one KV head; sampled sequences read its prefix
        B, hq, hkv, cap = 64, 64, 4, 131072
        _DATA["ga_decode"] = dict(kc=r.standard_normal((1, cap, 1, DQK)), vc=r.standard_normal((1, cap, 1, DV)),
                                  q=r.standard_normal((B, hq, DQK)), sink=r.standard_normal(hq),
                                  lengths=r.integers(4096, cap + 1, size=B), B=B, hq=hq, hkv=hkv)
    if "sparse_decode" in names:
        # the cache rows the key sets touch, drawn directly: [B, Hkv, 128 + 1024, D]
        B, hq, hkv, L, recent, n_sel = 8, 64, 4, 262144, 128, 1024
        sel = np.stack([np.stack([np.sort(r.choice(L - recent, n_sel, replace=False)) for _ in range(hkv)])
                        for _ in range(B)])
        _DATA["sparse_decode"] = dict(q=r.standard_normal((B, hq, DQK)), sink=r.standard_normal(hq), sel=sel,
                                      krows=r.standard_normal((B, hkv, recent + n_sel, DQK)),
                                      vrows=r.standard_normal((B, hkv, recent + n_sel, DV)),
                                      B=B, hq=hq, hkv=hkv, L=L, recent=recent, n_sel=n_sel)


# ----------------------------------------------------------------------------- worker tasks
def _task(args):
    """Runs one share of a workload; returns (work units, oracle seconds)."""
    name, part, nparts, limit = args
    d = _DATA[name]
    if name == "tiny_prefill":
        rows = [(0, h, i) for i in range(1024) for h in range(8)][part::nparts]
        t0 = time.perf_counter()
        ref.prefill(d["q"], d["k"], d["v"], d["sink"], 128, 1e4, 64, rows=rows)
        dt = time.perf_counter() - t0
        return sum(min(i + 1, 128) for (_, _, i) in rows) * FLOP_PER_PAIR, dt
    if name in ("swa_prefill", "ga_prefill"):
        n, hq, hkv, window, theta = d["n"], d["hq"], d["hkv"], d["window"], d["theta"]
        group = hq // hkv
        r = _rng(d["qseed"] + part)
        work, spent = 0.0, 0.0
        while spent < limit:                         # rows until this share's time is used
            i = int(r.integers(0, n))
            h = int(r.integers(0, hq))
            qrow = r.standard_normal(DQK)
            t1 = time.perf_counter()
            qr = ref.rope(qrow[None, None, :], np.array([float(i)]), theta, 64)[0, 0]
            keys = ref.window_keys(i, window, n)
            ref.attend_row(qr, d["kr"][:, h // group, :], d["v"][:, h // group, :], keys, d["sink"][h],
                           1.0 / math.sqrt(DQK))
            spent += time.perf_counter() - t1
            work += len(keys) * FLOP_PER_PAIR
        return work, spent
    if name == "swa_decode":
        bs = list(range(d["q"].shape[0]))[part::nparts]
        t0 = time.perf_counter()
        ref.decode(d["q"][bs], d["kc"][bs], d["vc"][bs], "ring", d["lengths"][bs], d["sink"])
        dt = time.perf_counter() - t0
        return len(bs) * 128 * 8 * BYTES_PER_KEY, dt
    if name == "ga_decode":
        hq, hkv = d["hq"], d["hkv"]
        group = hq // hkv
        r = _rng(4000 + part)
        work, t0 = 0.0, time.perf_counter()
        while time.perf_counter() - t0 < limit:      # (sequence, KV head) units until time is used
            b = int(r.integers(0, d["B"]))
            g = int(r.integers(0, hkv))
            L = int(d["lengths"][b])
            ref.decode(d["q"][b:b + 1, g * group:(g + 1) * group], d["kc"][:, :L], d["vc"][:, :L], "linear",
                       [L], d["sink"][g * group:(g + 1) * group])
            work += L * BYTES_PER_KEY
        return work, time.perf_counter() - t0
    if name == "sparse_decode":
        B, hq, hkv = d["B"], d["hq"], d["hkv"]
        group = hq // hkv
        units = [(b, g) for b in range(B) for g in range(hkv)][part::nparts]
        t0 = time.perf_counter()
        for b, g in units:
            keys = ref.sparse_key_set(d["L"], d["recent"], d["sel"][b, g])
            assert len(keys) == d["recent"] + d["n_sel"]
            for h in range(g * group, (g + 1) * group):
                ref.attend_row(d["q"][b, h], d["krows"][b, g], d["vrows"][b, g], np.arange(len(keys)),
                               d["sink"][h], 1.0 / math.sqrt(DQK))
        dt = time.perf_counter() - t0
        return len(units) * (d["recent"] + d["n_sel"]) * BYTES_PER_KEY, dt
    raise ValueError(name)


# full-workload sizes, for extrapolating the sampled ones
def _full_work(name):
    if name == "swa_prefill":
        return _swa_pairs(32768, 128) * 64 * FLOP_PER_PAIR
    if name == "ga_prefill":
        return _swa_pairs(32768, 0) * 64 * FLOP_PER_PAIR
    if name == "ga_decode":
        return float(np.sum(_DATA["ga_decode"]["lengths"])) * 4 * BYTES_PER_KEY
    return None


FULL = ("tiny_prefill", "swa_decode", "sparse_decode")
UNITS = {"tiny_prefill": "TFLOP/s", "swa_prefill": "TFLOP/s", "ga_prefill": "TFLOP/s",
         "swa_decode": "GB/s", "ga_decode": "GB/s", "sparse_decode": "GB/s"}


def run(names, cores, budget):
    """Times each workload on a fork pool of ``cores`` workers; returns a dict per workload."""
    _build(names)
    out = {}
    ctx = mp.get_context("fork")
    with ctx.Pool(cores) as pool:
        pool.map(abs, range(cores))                  # all workers up before the first timing
        for name in names:
            t0 = time.perf_counter()
            res = pool.map(_task, [(name, p, cores, budget) for p in range(cores)])
            wall = time.perf_counter() - t0
            work = sum(w for w, _ in res)
            scale = 1e12 if UNITS[name] == "TFLOP/s" else 1e9
            rate = work / wall / scale
            rec = {"rate": rate, "unit": UNITS[name], "wall_s": round(wall, 3)}
            if name in FULL:
                rec["s"] = round(wall, 3)
                rec["how"] = "full"
            else:
                full = _full_work(name)
                if name in ("swa_prefill", "ga_prefill"):
                    full_s = full / (work / wall) + _DATA[name]["t_rope"]   # plus the one K rotation
                else:
                    full_s = full / (work / wall)
                rec["s"] = round(full_s, 2)
                rec["how"] = "extrapolated"
                rec["sample_frac"] = round(work / full, 6)
            out[name] = rec
    return out


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--budget", type=float, default=3.0, help="seconds per sampled workload")
    ap.add_argument("--only", default=None)
    ap.add_argument("--cores", type=int, default=0)
    ap.add_argument("--steps", type=int, default=1)
    ap.add_argument("--warmup", type=int, default=0)
    args = ap.parse_args()
    avail = len(os.sched_getaffinity(0))
    cores = args.cores if args.cores > 0 else avail
    names = [args.only] if args.only else list(UNITS)
    if args.steps > 1 or args.warmup > 0:
        # repeated timings of one workload (the benchmark's reference arm)
        _build(names)
        ctx = mp.get_context("fork")
        steps = []
        with ctx.Pool(cores) as pool:
            pool.map(abs, range(cores))
            for s in range(args.warmup + args.steps):
                t0 = time.perf_counter()
                res = pool.map(_task, [(names[0], p, cores, args.budget) for p in range(cores)])
                wall = time.perf_counter() - t0
                if s >= args.warmup:
                    steps.append((sum(w for w, _ in res), wall))
        json.dump({"cores": cores, "available": avail, "steps": steps, "unit": UNITS[names[0]]}, sys.stdout)
        print()
        return
    res = run(names, cores, args.budget)
    json.dump({"cores": cores, "available": avail, "workloads": res}, sys.stdout)
    print()


if __name__ == "__main__":
    main()

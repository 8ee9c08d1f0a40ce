"""Multi-process plumbing for weak-scaling runs (one process per GPU).

Attention over independent (sequence, KV-head) units needs no exchange, so ranks
run independent problems; the only collectives are the timing barrier and the
max-over-ranks reduction of the measured time. Works with NCCL (GPU) and gloo
(CPU tests).
"""

from __future__ import annotations

import os

import torch
import torch.distributed as dist


def env_world():
    return int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def init(backend: str, timeout_s: float = 120.0):
    """Initialise the default process group from torchrun's environment (no-op at N=1)."""
    world, rank, _ = env_world()
    if world > 1 and not dist.is_initialized():
        from datetime import timedelta
        dist.init_process_group(backend=backend, timeout=timedelta(seconds=timeout_s))
    return world, rank


def shard_range(n_units: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous block [lo, hi) of ``n_units`` for ``rank`` (sizes differ by at most 1)."""
    base, extra = divmod(n_units, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def unit_shard(batch: int, n_kv_heads: int, rank: int, world: int) -> list[tuple[int, int]]:
    """This rank's (sequence, KV head) units of a decode call: a contiguous block of the
    flattened (b, g) order. Units share nothing, so a rank computes its block alone: the
    query heads of KV head g, its cache rows and its outputs (the partition is exact)."""
    lo, hi = shard_range(batch * n_kv_heads, rank, world)
    return [divmod(u, n_kv_heads) for u in range(lo, hi)]


def barrier():
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of a per-rank float across ranks (the job's time is the slowest rank's)."""
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, device=None) -> float:
    if not dist.is_initialized():
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def finalize():
    if dist.is_initialized():
        dist.destroy_process_group()

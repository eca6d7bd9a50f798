"""Multi-process plumbing: one process per GPU, no collective on the data path.

Attention heads are independent (the selection mask, the quantisation scales
and the output are all per head), so a forward pass shards by (batch, kv-head
group) with no exchange.  torch.distributed is used only for the barrier and
the max-over-ranks timing of the benchmark (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

import dataclasses
import datetime
import os
from typing import List, Optional, Tuple

import torch
import torch.distributed as dist


def env_ranks() -> Tuple[int, int, int]:
    """(rank, world_size, local_rank) from the launcher's environment (defaults: single process)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init(device: Optional[torch.device] = None, timeout_s: int = 120) -> bool:
    """Join the process group when running under torchrun; returns whether it did."""
    _, world, _ = env_ranks()
    if world <= 1 or dist.is_initialized():
        return dist.is_initialized()
    backend = "nccl" if device is not None and device.type == "cuda" else "gloo"
    kwargs = dict(backend=backend, timeout=datetime.timedelta(seconds=timeout_s))
    if backend == "nccl":
        kwargs["device_id"] = device
    dist.init_process_group(**kwargs)
    return True


def barrier() -> None:
    if dist.is_initialized():
        dist.barrier()


def max_over_ranks(value: float, device: Optional[torch.device] = None) -> float:
    """The largest value over all ranks (the job's time is its slowest rank's)."""
    if not dist.is_initialized():
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_heads(B: int, Hq: int, Hkv: int, rank: int, world: int) -> List[Tuple[int, int, int]]:
    """Split the (batch, kv head) units of one problem over ranks, contiguously.

    Each unit is one kv head with its Hq/Hkv query heads, so a rank's share is a
    self-contained attention problem.  Returns (b, hkv_begin, hkv_end) ranges.
    """
    units = B * Hkv
    lo = units * rank // world
    hi = units * (rank + 1) // world
    out = []
    u = lo
    while u < hi:
        b, h = divmod(u, Hkv)
        end = min(hi - b * Hkv, Hkv)
        out.append((b, h, end))
        u = b * Hkv + end
    return out


def finalize() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()


def rank_workload(w, rank: int):
    """The independent problem rank `rank` runs under weak scaling: same shape, own seed."""
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 7919 * rank)

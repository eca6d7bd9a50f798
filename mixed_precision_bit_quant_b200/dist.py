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


def shard_views(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor, rank: int, world: int):
    """The sub-problems rank `rank` of `world` owns in one attention problem.

    One (batch entry, range of kv heads) per item, with the Hq/Hkv query heads
    of each kv head: q[b, G*h0:G*h1], k/v[b, h0:h1] and o[b, G*h0:G*h1] are
    contiguous views of the caller's head-major tensors (no copy), and each
    item is a complete attention problem of its own (selection, scales and
    output are per head).  Returns a list of (q_view, k_view, v_view, o_view).
    """
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = []
    for b, h0, h1 in shard_heads(B, Hq, Hkv, rank, world):
        views = (q[b:b + 1, G * h0:G * h1], k[b:b + 1, h0:h1], v[b:b + 1, h0:h1], o[b:b + 1, G * h0:G * h1])
        assert all(t.is_contiguous() for t in views)
        out.append(views)
    return out


def attention_shard(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool, rank: int, world: int,
                    budget_bp: int = 500, budget_tiles: int = 0, o: Optional[torch.Tensor] = None,
                    mode: str = "score", fmt: str = "nvfp4") -> torch.Tensor:
    """This rank's share of one forward pass: quantize -> select -> mixed attention on each of
    its sub-problems (``shard_views``), written into its slices of ``o`` (allocated when None;
    the other ranks' slices are left as they are).  No collective: a caller that wants the
    whole O on one device gathers the slices itself.  Every rank's result equals the same
    rows of the unsharded call bit for bit, because every quantity is per head."""
    from . import _lib as L
    if o is None:
        o = torch.empty_like(q)
    for qv, kv, vv, ov in shard_views(q, k, v, o, rank, world):
        quant = L.quantize(qv, kv, vv, causal, fmt=fmt)
        mask, _ = L.select(qv, kv, causal, budget_bp, budget_tiles, mode=mode)
        L.attn_fwd(qv, kv, quant, mask, causal, o=ov)
    return o


def finalize() -> None:
    if dist.is_initialized():
        dist.destroy_process_group()


def rank_workload(w, rank: int):
    """The independent problem rank `rank` runs under weak scaling: same shape, own seed."""
    return w if rank == 0 else dataclasses.replace(w, seed=w.seed + 7919 * rank)

"""Timing helper for the benchmark's CPU baseline: the oracle on one sampled query tile.

TEST INFRASTRUCTURE (see ``oracle/formats.py``): only the benchmark's
CPU-baseline leg and the reference arm use this module.  It lives here, not
in bench.py, so that a spawned worker process can import it by name.
"""
from __future__ import annotations

import time


def tile_problem_time(args):
    """(seconds, FLOPs) of the oracle on one query tile of a single-head problem.

    ``args`` = (causal, budget_bp, budget_tiles, q, k, v, i): q[1,1,N,d] and k, v
    [1,1,N,d] hold one query head and its kv head; the oracle selects the tile's
    BF16 pairs (pool, score, top-k) and runs the mixed attention of query tile i
    with on-demand quantisation of the head, single-threaded.  FLOPs are the
    causal-adjusted attention FLOPs of the tile's rows.
    """
    from threadpoolctl import threadpool_limits

    from . import attention as oatt
    from . import select as osel
    causal, bp, bt, q, k, v, i = args
    N, d = int(q.shape[2]), int(q.shape[3])
    t0 = time.perf_counter()
    with threadpool_limits(limits=1):
        sel = osel.select(q, k, causal, bp, bt, rows=[(0, 0, i)])
        oatt.attn_forward(q, k, v, None, sel["mask"], causal, tiles=[(0, 0, i)])
    dt = time.perf_counter() - t0
    flops = 0.0
    for r in range(i * 128, min(N, (i + 1) * 128)):
        flops += 4.0 * d * ((r + 1) if causal else N)
    return dt, flops

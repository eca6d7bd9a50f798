"""The N>1 plumbing on CPU: two gloo ranks in separate processes.

Covers what bench.py does across ranks (process-group start from the
launcher's environment, barrier, max-over-ranks of a device time, each rank's
own independent problem) and the head sharding of one problem over ranks.  The
data path has no collective, so nothing else crosses ranks.
"""
import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

from mixed_precision_bit_quant_b200 import dist as mdist, workloads

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    assert mdist.env_ranks() == (rank, world, rank)
    assert mdist.init(None, timeout_s=60)
    mdist.barrier()
    local_ms = [3.5, 7.25][rank]                      # the slower rank sets the job's time
    job_ms = mdist.max_over_ranks(local_ms)
    w = mdist.rank_workload(workloads.WORKLOADS["tiny"], rank)
    q, _, _ = workloads.generate(w)
    mdist.barrier()
    mdist.finalize()
    with open(os.path.join(outdir, f"r{rank}.json"), "w") as f:
        json.dump({"job_ms": job_ms, "seed": w.seed, "q0": float(q.flatten()[:64].float().sum())}, f)


def test_two_gloo_ranks_barrier_and_max_over_ranks(tmp_path):
    mp.start_processes(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    r = [json.load(open(tmp_path / f"r{i}.json")) for i in range(2)]
    assert r[0]["job_ms"] == r[1]["job_ms"] == 7.25
    assert r[0]["seed"] != r[1]["seed"] and r[0]["q0"] != r[1]["q0"]    # independent problems


@pytest.mark.parametrize("B,Hkv,world", [(1, 8, 2), (1, 8, 3), (2, 8, 3), (3, 2, 4), (1, 1, 2), (4, 8, 8)])
def test_shard_heads_covers_every_unit_once(B, Hkv, world):
    seen = []
    for rank in range(world):
        for b, h0, h1 in mdist.shard_heads(B, 4 * Hkv, Hkv, rank, world):
            assert 0 <= b < B and 0 <= h0 < h1 <= Hkv
            seen += [(b, h) for h in range(h0, h1)]
    assert sorted(seen) == [(b, h) for b in range(B) for h in range(Hkv)]
    assert len(seen) == len(set(seen))


def test_reference_arm_under_two_ranks_prints_once():
    """`bench.py --impl reference` under torchrun: rank 0 prints one line, rank 1 exits 0 without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}", os.path.join(ROOT, "bench.py"),
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "0", "--workload", "tiny"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [json.loads(x) for x in p.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    ln = lines[0]
    assert ln["impl"] == "reference" and ln["n_gpus"] == 2 and ln["value"] > 0
    assert ln["e2e"]["h2d_bytes_per_step"] == 0 and ln["cpu_baseline"]["kind"] == "oracle"


def _shard_worker(rank, world, port, outdir):
    """Each rank fills its shard_views slices of O with rank-specific values; a gloo
    all-gather (test only) reassembles the whole O, which must carry every head once."""
    import torch
    import torch.distributed as tdist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    mdist.init(None, timeout_s=60)
    B, Hq, Hkv, N, d = 3, 8, 4, 5, 4
    q = torch.zeros(B, Hq, N, d)
    k = torch.zeros(B, Hkv, N, d)
    o = torch.full((B, Hq, N, d), -1.0)
    for qv, kv, vv, ov in mdist.shard_views(q, k, k, o, rank, world):
        ov.fill_(float(rank))
    parts = [torch.empty_like(o) for _ in range(world)]
    tdist.all_gather(parts, o)
    mdist.finalize()
    owner = torch.full((B, Hq), -1.0)
    for r, part in enumerate(parts):
        mine = (part[:, :, 0, 0] == r)
        assert bool((owner[mine] == -1).all())         # no head filled by two ranks
        owner[mine] = r
    with open(os.path.join(outdir, f"s{rank}.json"), "w") as f:
        json.dump(owner.tolist(), f)


@pytest.mark.parametrize("world", [2, 3])
def test_shard_views_partition_and_reassembly(tmp_path, world):
    mp.start_processes(_shard_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    owners = [json.load(open(tmp_path / f"s{r}.json")) for r in range(world)]
    assert all(ow == owners[0] for ow in owners)
    flat = [x for row in owners[0] for x in row]
    assert -1 not in flat                                     # every head owned
    G = 2
    for row in owners[0]:                                     # a GQA group never splits
        assert all(row[G * i] == row[G * i + 1] for i in range(len(row) // G))

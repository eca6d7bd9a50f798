"""Benchmark: mixed FP4/BF16 attention forward (prefill) on B200.

One step = the whole hot path on one batch of synthetic input resident in
HBM: thrift_quantize -> thrift_select -> thrift_attn_fwd.  Default workload:
causal GQA prefill, B=1, Hq=32, Hkv=8, N=32768, d=128, 5% BF16 tile budget.

Metric: effective attention TFLOP/s, causal-adjusted (2*B*Hq*N^2*d FLOPs per
step for causal runs, 4*B*Hq*N^2*d otherwise) over the device-timed step.

Multi-GPU (torchrun, one process per GPU): every rank runs its own full
problem (heads and batches are independent; no collective on the data
path), so scaling is weak and value = all ranks' FLOPs / max-over-ranks time.

`--impl reference` times the CPU oracle (the statement of the method the
library is checked against) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from mixed_precision_bit_quant_b200 import dist as mdist, workloads  # noqa: E402

METRIC = "attn TFLOPS (causal-adj) & % of mixed FP4/BF16 roofline, N=32K, 5% BF16"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def hi_lo_pairs(w: workloads.Workload):
    """(BF16 pairs, FP4 pairs) the budget rule yields for workload w (closed form)."""
    T = w.T
    hi = lo = 0
    for i in range(T):
        n_i = i + 1 if w.causal else T
        nf = 1 if i == 0 else 2
        if w.budget_tiles > 0:
            k = min(n_i, max(nf, w.budget_tiles))
        elif w.budget_bp <= 0:
            k = 0
        elif w.budget_bp >= 10000:
            k = n_i
        else:
            k = min(n_i, max(nf, (w.budget_bp * n_i + 9999) // 10000))
        hi += k
        lo += n_i - k
    return hi * w.B * w.Hq, lo * w.B * w.Hq


def attn_roofline(w: workloads.Workload, peaks: dict, key: str = "bf16_tflops"):
    """Mixed tensor roofline of the attention kernel.

    Per computed 128x128 tile pair: F = 2*128*128*d FLOPs for Q K^T and the
    same for P V.  FP4 pairs run Q K^T at the FP4 rate and P V at the FP8
    rate; BF16 pairs run both at the BF16 rate.  Rates: the measured BF16
    GEMM peak, times 2 (FP8) and 4 (FP4), the nominal dense ratios.
    """
    hi, lo = hi_lo_pairs(w)
    F = 2.0 * 128 * 128 * w.d
    p16 = peaks[key] * 1e12
    p8, p4 = 2 * p16, 4 * p16
    t = lo * (F / p4 + F / p8) + hi * (2 * F / p16)
    t_fp4_both = lo * (2 * F / p4) + hi * (2 * F / p16)  # stricter: P V at the FP4 rate too
    flops = (hi + lo) * 2 * F
    return dict(flops=flops, t_roof=t, peak=flops / t, hi=hi, lo=lo, t_roof_fp4_both=t_fp4_both)


SPEC_PEAKS_TFLOPS = {"fp4": 9000.0, "fp8": 4500.0, "bf16": 2250.0}   # B200 dense, nominal


def attn_roofline_rates(w: workloads.Workload, p4: float, p8: float, p16: float):
    """Roofline time of the attention kernel for explicit per-precision rates (TFLOP/s)."""
    hi, lo = hi_lo_pairs(w)
    F = 2.0 * 128 * 128 * w.d
    return (lo * (F / (p4 * 1e12) + F / (p8 * 1e12)) + hi * (2 * F / (p16 * 1e12)),
            lo * (2 * F / (p4 * 1e12)) + hi * (2 * F / (p16 * 1e12)))


def measure_mma_rates(mq) -> dict:
    """Dense TFLOP/s of the three tensor-core instruction forms the attention kernel issues
    (thrift_probe_mma, one CTA per SM): NVFP4 block-scaled Q.K^T, e4m3 P.V with P in tensor
    memory, BF16 Q.K^T, each 128 x 128 x 128 per step."""
    out = {}
    for name, kind, iters in (("fp4", 0, 20000), ("fp8", 1, 10000), ("bf16", 2, 4000)):
        mq.probe_mma(kind, 128, 200)
        r = mq.probe_mma(kind, 128, iters)
        out[name] = r["tflops"]
        out[name + "_flop_per_clk_per_sm"] = r["flop_per_clk_per_sm"]
    return out


def attn_algorithmic_bytes(w: workloads.Workload, hi: int, lo: int) -> float:
    """Compulsory HBM bytes of one attention launch (each operand read once, O written once)."""
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    q = B * Hq * N * d * (2 + 0.5 + 1 / 16)
    kv = B * Hkv * N * d * (2 + 0.5 + 1 / 16 + 1 + 2)
    o = B * Hq * N * d * 2
    return q + kv + o


def profiled_traffic(kernel_source: str, summary: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on this source."""
    import hashlib
    try:
        with open(kernel_source, "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        fields = {}
        with open(summary) as f:
            for ln in f:
                if ":" in ln:
                    k, _, v = ln.strip().partition(":")
                    fields[k.strip()] = v.strip()
        if fields.get("attn_fwd_source_sha256") == sha:
            return float(fields["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError):
        pass
    return None


def quantize_algorithmic_bytes(w):
    B, Hq, Hkv, N, d = w.B, w.Hq, w.Hkv, w.N, w.d
    Np = w.T * 128
    inp = (B * Hq + 2 * B * Hkv) * N * d * 2
    out = (B * Hq + B * Hkv) * (N * d / 2 + N * d / 16 + w.T * 128 * d / 16) + B * Hkv * d * Np * 3
    return inp + out


def select_algorithmic_bytes(w):
    return (w.B * w.Hq + w.B * w.Hkv) * w.N * w.d * 2


class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in a background process."""

    FIELDS = ("index,timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t_start = self.t_stop = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self._th = threading.Thread(target=self._read, daemon=True)
        self._th.start()

    def _read(self):
        for ln in self.proc.stdout:
            self.lines.append((time.time(), ln.strip()))

    def mark_start(self):
        self.t_start = time.time()

    def mark_stop(self):
        self.t_stop = time.time()

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        inwin = [(t, l) for (t, l) in self.lines if self.t_start - 0.05 <= t <= self.t_stop + 0.15]
        if not inwin:
            # nearest sample to the window's middle
            mid = 0.5 * (self.t_start + self.t_stop)
            inwin = [min(self.lines, key=lambda x: abs(x[0] - mid))]
        sms, maxs, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, l in inwin:
            f = [x.strip() for x in l.split(",")]
            try:
                sms.append(float(f[2]))
                maxs.append(float(f[3]))
                power.append(float(f[4]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, f[6:10]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sms) if sms else None, "sm_max_mhz": max(maxs) if maxs else None,
                "power_w_max": max(power) if power else None, "reasons": sorted(reasons), "samples": len(sms)}


def oracle_sample_run(w: workloads.Workload, q, k, v, tiles):
    """Time the CPU oracle on `tiles`: for each (b, h, i), the single-head problem
    (q head h, its kv head) runs select + mixed attention with on-demand
    quantisation.  Heads are independent, so this is the same arithmetic as
    the full problem restricted to those rows.  Single-threaded BLAS."""
    from threadpoolctl import threadpool_limits

    from oracle import attention as oatt
    from oracle import select as osel
    G = w.Hq // w.Hkv
    t0 = time.perf_counter()
    with threadpool_limits(limits=1):
        for (b, h, i) in tiles:
            qs = q[b:b + 1, h:h + 1]
            ks = k[b:b + 1, h // G:h // G + 1]
            vs = v[b:b + 1, h // G:h // G + 1]
            sel = osel.select(qs, ks, w.causal, w.budget_bp, w.budget_tiles, rows=[(0, 0, i)])
            oatt.attn_forward(qs, ks, vs, None, sel["mask"], w.causal, tiles=[(0, 0, i)])
    dt = time.perf_counter() - t0
    flops = 0.0
    for (_, _, i) in tiles:
        r0, r1 = i * 128, min(w.N, (i + 1) * 128)
        for r in range(r0, r1):
            flops += 4.0 * w.d * ((r + 1) if w.causal else w.N)
    return dt, flops


def cpu_baseline(w, q, k, v, n_tiles: int, seed: int = 1, procs: int = 0):
    """The oracle on sampled query tiles: one core, and (procs > 1) a spawned process pool
    over the host's cores; the full problem's time is extrapolated from the FLOP rate."""
    tiles = workloads.sample_query_tiles(w, n_tiles, seed=seed)
    dt, flops = oracle_sample_run(w, q, k, v, tiles)
    one = flops / dt / 1e12
    full_flops = w.causal_adjusted_flops()
    out = {"value": one, "unit": UNIT, "cores": 1, "kind": "oracle",
           "sample": f"{len(tiles)} query tiles (seed {seed}) of {w.name}, each as its single-head problem: "
                     f"pool/score/select + quantise the head + mixed attention of the tile; "
                     f"{dt:.1f} s, single-threaded numpy (FP32 decisions, FP64 attention)",
           "seconds": dt, "extrapolated_full_problem_s_one_core": full_flops / (one * 1e12)}
    if procs > 1:
        import torch.multiprocessing as tmp
        from oracle.timing import tile_problem_time
        G = w.Hq // w.Hkv
        ptiles = workloads.sample_query_tiles(w, procs * 2, seed=seed + 100)
        for t in (q, k, v):
            t.share_memory_()        # workers receive views of the same host memory, no copies
        jobs = [(w.causal, w.budget_bp, w.budget_tiles, q[b:b + 1, h:h + 1], k[b:b + 1, h // G:h // G + 1],
                 v[b:b + 1, h // G:h // G + 1], i) for (b, h, i) in ptiles]
        ctx = tmp.get_context("spawn")
        with ctx.Pool(procs) as pool:
            pool.map(tile_problem_time, jobs[:procs], chunksize=1)   # import and warm every worker
            t0 = time.perf_counter()
            res = pool.map(tile_problem_time, jobs, chunksize=1)
            wall = time.perf_counter() - t0
        pflops = sum(f for _, f in res)
        allc = pflops / wall / 1e12
        out.update({"value": allc, "cores": procs, "single_core_value": one,
                    "sample": f"{len(jobs)} query tiles (seed {seed + 100}) of {w.name} on a spawned pool of "
                              f"{procs} processes (one BLAS thread each), {wall:.1f} s wall; single core: "
                              f"{len(tiles)} tiles, {dt:.1f} s",
                    "extrapolated_full_problem_s": full_flops / (allc * 1e12)})
    return out


def run_reference(args, w):
    rank, world, _ = mdist.env_ranks()
    if rank != 0:
        return 0
    q, k, v = workloads.generate(w)
    vals = []
    cb = None
    n_tiles = args.ref_tiles
    for s in range(args.warmup + args.steps):
        tiles = workloads.sample_query_tiles(w, n_tiles, seed=1 + s)
        dt, flops = oracle_sample_run(w, q, k, v, tiles)
        if s >= args.warmup:
            vals.append((dt, flops))
    tot_t = sum(d for d, _ in vals)
    tot_f = sum(f for _, f in vals)
    value = tot_f / tot_t / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_t / max(1, len(vals)),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_of(w, world),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": f"{n_tiles} query tiles per step (seeds 1..), select + mixed attention"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_decode(args):
    """Decode-step measurement (not the headline): one step of one query token per sequence
    against per-token MXFP4 / MXFP8 caches of `--decode-len` tokens (sink and window in BF16),
    B=8, Hq=32, Hkv=8, d=128.  Reports the step's HBM bytes (quantised cache rows, BF16 sink and
    window rows, query, output and the per-chunk softmax states written and read back) over its
    CUDA-event time, against the measured HBM copy bandwidth.  The caches (0.4 GB at 32K) exceed
    L2, so no flush is needed between steps."""
    import mixed_precision_bit_quant_b200 as mq
    rank, world, local = mdist.env_ranks()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    peaks, peak_src = _peaks()
    B, Hq, Hkv, L, d = 8, 32, 8, args.decode_len, 128
    g = torch.Generator().manual_seed(3)
    q = torch.randn((B, Hq, d), generator=g).to(torch.bfloat16).to(dev)
    k = (torch.randn((B, Hkv, L, d), generator=g) + 2.0 * torch.randn((B, Hkv, 1, d), generator=g)).to(torch.bfloat16)
    k[:, :, 0] *= 8
    k = k.to(dev)
    v = torch.randn((B, Hkv, L, d), generator=g).to(torch.bfloat16).to(dev)
    cache = mq.decode_quantize_cache(k, v)
    o = torch.empty_like(q)
    ws = None
    mq.decode_step(q, k, v, cache, o=o)
    torch.cuda.synchronize(dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    for _ in range(args.warmup):
        mq.decode_step(q, k, v, cache, o=o)
    torch.cuda.synchronize(dev)
    e0, e1 = ev(), ev()
    e0.record()
    for _ in range(args.steps):
        mq.decode_step(q, k, v, cache, o=o)
    e1.record()
    torch.cuda.synchronize(dev)
    st, word = mq.device_status()
    if st != 0:
        raise RuntimeError(f"device watchdog raised {word:#x}")
    ms = e0.elapsed_time(e1) / args.steps
    hp = min(L, 256)
    nchunk = (L + 255) // 256
    byts = (B * Hkv * (L - hp) * (d // 2 + d // 32 + d + d // 32) + B * Hkv * hp * d * 2 * 2
            + B * Hq * d * 2 * 2 + 2 * B * Hq * nchunk * (2 + d) * 4)
    gbs = byts / (ms * 1e-3) / 1e9
    print(json.dumps({"metric": "decode step HBM GB/s (per-token MXFP4 K / MXFP8 V cache, BF16 sink + window)",
                      "value": gbs, "unit": "GB/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
                      "n_gpus": 1, "config": {"workload": f"decode B={B} Hq={Hq} Hkv={Hkv} L={L} d={d}"},
                      "roofline": {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                                   "frac": gbs / peaks["hbm_gbs"], "bytes_per_step": byts,
                                   "peak_source": peak_src}}), flush=True)
    return 0


def config_of(w, world):
    return {"workload": f"{w.name}: causal={int(w.causal)} B={w.B} Hq={w.Hq} Hkv={w.Hkv} N={w.N} d={w.d} "
                        f"budget_bp={w.budget_bp} budget_tiles={w.budget_tiles}",
            "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "N": w.N, "d": w.d, "causal": w.causal,
            "budget_bp": w.budget_bp, "parallelism": f"independent problem per rank x{world}",
            "l2": "inputs larger than L2 (Q alone is 268 MB at N=32K); no flush between steps"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="thrift", choices=["thrift", "reference"])
    ap.add_argument("--workload", default="llm32k", choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--budget-bp", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--cpu-tiles", type=int, default=16)
    ap.add_argument("--ref-tiles", type=int, default=1)
    ap.add_argument("--cpu-procs", type=int, default=-1, help="oracle pool size (-1: the host's cores, at most 32)")
    ap.add_argument("--fmt", default="nvfp4", choices=["nvfp4", "mxfp4"])
    ap.add_argument("--mode", default="score", choices=["score", "vertical"])
    ap.add_argument("--no-mma-probe", action="store_true")
    ap.add_argument("--decode", action="store_true", help="measure the decode step instead (not the headline)")
    ap.add_argument("--decode-len", type=int, default=32768)
    args = ap.parse_args()
    if args.decode:
        return run_decode(args)
    w = workloads.WORKLOADS[args.workload]
    if args.budget_bp is not None:
        w = w.with_budget(bp=args.budget_bp)
    if args.impl == "reference":
        return run_reference(args, w)

    import mixed_precision_bit_quant_b200 as mq

    rank, world, local = mdist.env_ranks()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    mdist.init(dev)
    peaks, peak_src = _peaks()

    # weak scaling: each rank owns an independent problem of the same shape (its own seed)
    q_h, k_h, v_h = workloads.generate(mdist.rank_workload(w, rank))
    q, k, v = (t.to(dev) for t in (q_h, k_h, v_h))
    quant = mq.alloc_quantized(mq.shape_of(q, k, w.causal), dev)
    shape = mq.shape_of(q, k, w.causal)
    ws_q = torch.empty(max(16, mq.workspace_bytes(shape, mq.OP_QUANTIZE)), dtype=torch.uint8, device=dev)
    ws_s = torch.empty(max(16, mq.workspace_bytes(shape, mq.OP_SELECT_VERTICAL)), dtype=torch.uint8, device=dev)
    T, W = w.T, (w.T + 31) // 32
    mask = torch.empty((w.B, w.Hq, T, W), dtype=torch.int32, device=dev)
    counts = torch.empty((w.B, w.Hq, T), dtype=torch.int32, device=dev)
    o = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    K = args.steps
    marks = [(ev(), ev(), ev(), ev()) for _ in range(K)]

    def step(m=None):
        if m is not None:
            m[0].record(stream)
        mq.quantize(q, k, v, w.causal, out=quant, ws=ws_q, fmt=args.fmt)
        if m is not None:
            m[1].record(stream)
        mq.select(q, k, w.causal, w.budget_bp, w.budget_tiles, mask=mask, counts=counts, ws=ws_s, mode=args.mode)
        if m is not None:
            m[2].record(stream)
        mq.attn_fwd(q, k, quant, mask, w.causal, o=o)
        if m is not None:
            m[3].record(stream)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    status, word = mq.device_status()
    if status != 0:
        raise RuntimeError(f"device watchdog raised {word:#x} during warm-up")

    sampler = None if args.no_clocks else ClockSampler(local)
    if sampler:
        sampler.start()
        time.sleep(0.6)  # nvidia-smi start-up
    mdist.barrier()
    torch.cuda.synchronize(dev)
    n0 = mq.launch_count()
    t_begin, t_end = ev(), ev()
    if sampler:
        sampler.mark_start()
    t_begin.record(stream)
    for s in range(K):
        step(marks[s])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    if sampler:
        sampler.mark_stop()
    mdist.barrier()
    launches = mq.launch_count() - n0
    status, word = mq.device_status()
    if status != 0:
        raise RuntimeError(f"device watchdog raised {word:#x} in the timed region")
    if sampler:
        time.sleep(0.2)
        sampler.stop()
    total_ms = mdist.max_over_ranks(t_begin.elapsed_time(t_end), dev)
    ms_step = total_ms / K
    # per-stage times: the median over the timed steps (the first step's quantize stage also
    # holds the host's enqueue latency after the synchronisation that opens the timed region)
    q_ms = statistics.median(m[0].elapsed_time(m[1]) for m in marks)
    s_ms = statistics.median(m[1].elapsed_time(m[2]) for m in marks)
    a_ms = statistics.median(m[2].elapsed_time(m[3]) for m in marks)

    eff_flops = w.causal_adjusted_flops()
    value = world * eff_flops / (ms_step * 1e-3) / 1e12
    roof = attn_roofline(w, peaks, "bf16_tflops")
    achieved = roof["flops"] / (a_ms * 1e-3) / 1e12
    peak = roof["peak"] / 1e12

    # ------------------------------------------------ end to end through host buffers
    # Every step copies Q, K, V from pinned host memory and O back.  The copies run on
    # their own streams and overlap the kernels of the neighbouring steps (the copy
    # engines work beside the SMs); two device buffer sets alternate between steps.
    e2e = None
    if not args.no_e2e:
        qp, kp, vp = (t.pin_memory() for t in (q_h, k_h, v_h))
        o_host = [torch.empty(q_h.shape, dtype=torch.bfloat16).pin_memory() for _ in range(2)]
        bufs = [(q, k, v, o), tuple(torch.empty_like(t) for t in (q, k, v, o))]
        s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        in_done = [torch.cuda.Event() for _ in range(2)]
        cmp_done = [torch.cuda.Event() for _ in range(2)]
        out_done = [torch.cuda.Event() for _ in range(2)]

        def run_step(qb, kb, vb, ob):
            mq.quantize(qb, kb, vb, w.causal, out=quant, ws=ws_q, fmt=args.fmt)
            mq.select(qb, kb, w.causal, w.budget_bp, w.budget_tiles, mask=mask, counts=counts, ws=ws_s,
                      mode=args.mode)
            mq.attn_fwd(qb, kb, quant, mask, w.causal, o=ob)

        ke = max(3, min(10, K))
        e0, e1 = ev(), ev()
        for it in range(2 + ke):
            if it == 2:
                torch.cuda.synchronize(dev)
                mdist.barrier()
                e0.record(s_in)
            bi = it % 2
            qb, kb, vb, ob = bufs[bi]
            with torch.cuda.stream(s_in):
                if it >= 2:
                    s_in.wait_event(cmp_done[bi])  # step it-2 has finished reading this buffer set
                qb.copy_(qp, non_blocking=True)
                kb.copy_(kp, non_blocking=True)
                vb.copy_(vp, non_blocking=True)
                in_done[bi].record(s_in)
            stream.wait_event(in_done[bi])
            if it >= 2:
                stream.wait_event(out_done[bi])  # step it-2's O has been read back
            run_step(qb, kb, vb, ob)
            cmp_done[bi].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(cmp_done[bi])
                o_host[bi].copy_(ob, non_blocking=True)
                out_done[bi].record(s_out)
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        e_ms = mdist.max_over_ranks(e0.elapsed_time(e1) / ke, dev)
        h2d = sum(t.numel() * t.element_size() for t in (q_h, k_h, v_h))
        e2e = {"value": world * eff_flops / (e_ms * 1e-3) / 1e12, "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": o_host[0].numel() * 2,
               "api": "mixed_precision_bit_quant_b200.quantize/select/attn_fwd (C ABI); pinned host copies "
                      "on their own streams, overlapping the neighbouring steps' kernels"}

    # tcgen05 rates of this GPU (after the timed region: the probe's launches are not counted)
    mma = None
    if not args.no_mma_probe:
        mma = measure_mma_rates(mq)
    spec_t, spec_t_fp4 = attn_roofline_rates(w, SPEC_PEAKS_TFLOPS["fp4"], SPEC_PEAKS_TFLOPS["fp8"],
                                             SPEC_PEAKS_TFLOPS["bf16"])
    roof_extra = {"frac_vs_spec_peaks": spec_t / (a_ms * 1e-3),
                  "frac_vs_spec_peaks_pv_at_fp4_rate": spec_t_fp4 / (a_ms * 1e-3),
                  "spec_peaks_tflops": SPEC_PEAKS_TFLOPS}
    if mma is not None:
        mt, mt_fp4 = attn_roofline_rates(w, mma["fp4"], mma["fp8"], mma["bf16"])
        roof_extra.update({"frac_vs_tcgen05_measured": mt / (a_ms * 1e-3),
                           "frac_vs_tcgen05_measured_pv_at_fp4_rate": mt_fp4 / (a_ms * 1e-3),
                           "tcgen05_measured_tflops": mma,
                           "t_roof_tcgen05_measured_ms": mt * 1e3})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        procs = args.cpu_procs if args.cpu_procs > 0 else min(32, os.cpu_count() or 1)
        cpu = cpu_baseline(w, q_h, k_h, v_h, args.cpu_tiles, procs=procs)

    traffic = None
    if w.name == "llm32k" and w.budget_bp == 500:
        traffic = profiled_traffic(os.path.join(ROOT, "mixed_precision_bit_quant_b200", "csrc", "attn_fwd.cu"),
                                   os.path.join(ROOT, "profiles", "attn_fwd_llm32k_5pct.md"))
    if rank == 0:
        hbm = peaks["hbm_gbs"]
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
            "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": f"{args.fmt}/e4m3/bf16 (fp32 accumulate)", "data": "synthetic",
            "config": dict(config_of(w, world), fmt=args.fmt, select_mode=args.mode),
            "roofline": {"bound": "tensor", "kernel": "attn_fwd_kernel<128>", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 {peaks['bf16_tflops']} TF/s burst; FP8 = 2x, FP4 = 4x "
                                        f"(nominal dense ratios); BF16 pairs {roof['hi']}, FP4 pairs {roof['lo']}",
                         "t_roof_ms": roof["t_roof"] * 1e3, "algorithmic_flops": roof["flops"],
                         "frac_if_pv_at_fp4_rate": roof["t_roof_fp4_both"] / (a_ms * 1e-3), **roof_extra},
            "stages_ms": {"quantize": q_ms, "select": s_ms, "attn_fwd": a_ms},
            "stages_gbs": {"quantize": quantize_algorithmic_bytes(w) / (q_ms * 1e-3) / 1e9,
                           "select": select_algorithmic_bytes(w) / (s_ms * 1e-3) / 1e9,
                           "hbm_peak": hbm},
            "attn_only_tflops_causal_adj": eff_flops / (a_ms * 1e-3) / 1e12,
            "attn_algorithmic_bytes": attn_algorithmic_bytes(w, roof["hi"], roof["lo"]),
            "gpu_launches": launches,
            "clocks": sampler.summary() if sampler else None,
            "e2e": e2e,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    mdist.finalize()
    return 0


if __name__ == "__main__":
    sys.exit(main())

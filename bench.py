#!/usr/bin/env python
"""Benchmark of the block-sparse attention path on B200.

One step = the whole prefill path over one batch of the 32K workload: block
statistics -> Taylor-score top-p selection -> block-sparse causal attention
(three kernels through the C-ABI). Printed as one JSON line by rank 0:

  value     prefill tokens/s over all ranks (device time, CUDA events on the
            launching stream, inputs resident in HBM, L2 flushed between steps)
  roofline  the attention kernel's kept-block TFLOP/s against the measured bf16
            tensor peak
  decode    decode kept-KV GB/s of the decode workload against measured HBM peak
  e2e       the same prefill metric through spa_prefill_host with pinned host
            buffers: the host -> device copies of Q, K, V and the device -> host
            copy of O inside the timed region, pipelined against the kernels over
            chunks of (b, kv-head) pairs
  diagnostics   per prefill workload (1K fp32, 8K, 32K): kept fraction of the
            causal blocks (mean, p50, p99), operator MSE against dense causal
            attention and the attention-mass coverage of the kept set, all from
            the library's own kernels (dense = the same prefill at top_p = 1)
  cpu_baseline  the CPU oracle on a bounded sample (rank 0, one GPU only)

`--impl reference` times the CPU oracle on the same workload instead (the
reference arm of this comparison) and prints the same line with "impl":
"reference".

Multi-GPU: one process per GPU (torchrun); each rank takes a contiguous share of
the workload's (b, kv-head) units, its kv-heads with their query heads (the units
are independent through every kernel, so the path needs no collective and the
output stays head-sharded); the time is the max over ranks and the value counts
every token of the job once (strong scaling). The legs beside the headline step
run on one GPU only.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from workloads import WORKLOADS, generate, n_threads  # noqa: E402

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
METRIC = "prefill tokens/s & kept-FLOP TFLOP/s at 32K; decode KV GB/s vs HBM peak"


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def captured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu capture of `kernel`, or None when
    the kernel's source changed since the capture (or none was taken)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            rec = json.load(f)[kernel]
        with open(os.path.join(ROOT, "block_sparse_long_stats_b200", "csrc", "prefill_tc.cu"), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
    except (OSError, KeyError, ValueError):
        return None
    if rec.get("source_sha256") != sha or rec.get("workload") != workload:
        return None
    return float(rec["dram_bytes_per_launch"])


# ---------------------------------------------------------------- algorithmic work

def kept_flops(count: np.ndarray, idx: np.ndarray, L: int, block: int, d: int) -> float:
    """4 d x (unmasked query-key pairs) over every kept (head, query block, block) tile."""
    nq = count.shape[-1]
    n_i = np.minimum(block, L - np.arange(nq) * block).astype(np.float64)       # rows per q-block
    last = np.take_along_axis(idx, np.maximum(count - 1, 0)[..., None], axis=-1)[..., 0]
    diag = (last == np.arange(nq)).astype(np.float64)
    pairs = (count - diag) * n_i * block + diag * n_i * (n_i + 1) / 2
    return float(4.0 * d * pairs.sum())


def kept_kv_bytes(count: np.ndarray, idx: np.ndarray, G: int, T: int, block: int, d: int) -> float:
    """K and V bytes of the union of the kept blocks of each (b, kv-head)."""
    B, Hq = count.shape[:2]
    nb = -(-T // block)
    tokens = np.minimum(block, T - np.arange(nb) * block)
    total = 0
    for b in range(B):
        for g in range(Hq // G):
            kept = np.zeros(nb, bool)
            for h in range(g * G, (g + 1) * G):
                kept[idx[b, h, 0, :count[b, h, 0]]] = True
            total += int(tokens[kept].sum())
    return float(total * d * 2 * 2)


def workload_config(w, n_gpus: int) -> dict:
    """The `config` of the JSON line, identical for the CUDA arm and the reference arm."""
    return {"workload": w.name, "B": w.B, "L": w.T, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d,
            "block": w.block, "top_p": w.top_p,
            "parallelism": "one GPU" if n_gpus == 1 else f"(b, kv-head) units split over {n_gpus} GPUs",
            "l2": "flushed between timed steps (256 MiB written, then 256 MiB of another buffer read)"}


class L2Flush:
    """Between timed steps: 256 MiB written (every line a step touched is evicted),
    then 256 MiB of a second buffer read, so that the next step starts on an L2 of
    clean lines. Without the read, up to 126 MB of the memset's dirty lines are
    written back while the step's first kernel runs and are charged to it (at 32K
    that doubled the DRAM traffic of the 25 us statistics launch)."""

    def __init__(self, torch):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(64 << 20, dtype=torch.int32, device="cuda")

    def zero_(self):
        self.w.zero_()
        self.r.amax()


# ---------------------------------------------------------------- ranks

def head_shard(B: int, Hkv: int, world: int, rank: int) -> tuple[int, int]:
    """The (b, kv-head) units rank `rank` of `world` takes: a contiguous share
    [u0, u1) of the B * Hkv units in (b, kv-head) order. Each unit is an independent
    problem through every kernel (its kv-head's statistics, its query heads'
    selection and attention), so a rank needs no other rank's data and the output
    stays head-sharded, as tensor-parallel attention keeps it."""
    U = B * Hkv
    return rank * U // world, (rank + 1) * U // world


def max_over_ranks(v: float, world: int, device) -> float:
    """Max of a per-rank device time over all ranks (all_reduce MAX; no-op on one rank)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: int, world: int, steps: int, total_ms: float) -> float:
    """Whole-job units/s: every rank processes its own replica (weak scaling), and the
    slowest rank's time counts."""
    return world * units_per_rank * steps / (total_ms / 1e3)


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.dev}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.15)
        self.proc.terminate()
        self.proc.wait()
        rows = [l.split(",") for l in open(self.path).read().strip().splitlines() if l.strip()]
        os.unlink(self.path)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            r = [c.strip() for c in r]
            try:
                sm.append(float(r[1]))
                mx.append(float(r[2]))
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle

def time_oracle(w, x, n_tokens: int, seed: int):
    """Oracle on a bounded sample: stats + selection on the whole workload, masked
    attention on n_tokens uniformly drawn query positions (all heads). Returns
    (tokens/s estimate, detail)."""
    import oracle
    t0 = time.perf_counter()
    sel = oracle.select(x["q"], x["k"], w.dtype, w.block, w.scale, w.top_p, w.n_sink, w.n_local,
                        w.k_min)
    t_sel = time.perf_counter() - t0
    rng = np.random.default_rng(seed)
    pos = rng.choice(w.B * w.Lq, size=n_tokens, replace=False)
    b, t = pos // w.Lq, pos % w.Lq
    rows = ((b[:, None] * w.Hq + np.arange(w.Hq)[None, :]) * w.Lq + t[:, None]).reshape(-1)
    t0 = time.perf_counter()
    oracle.attention(x["q"], x["k"], x["v"], w.dtype, w.block, sel["idx"], sel["count"], w.scale,
                     rows=rows)
    t_att = time.perf_counter() - t0
    total_tokens = w.B * w.Lq
    t_est = t_att + t_sel * n_tokens / total_tokens
    return n_tokens / t_est, {"t_select_s": t_sel, "t_attention_sample_s": t_att,
                              "threads": oracle.num_threads()}


# ---------------------------------------------------------------- reference arm

def run_reference(args, rank: int):
    if rank != 0:
        return
    w = WORKLOADS[args.workload]
    x = generate(w)
    per_step = []
    n_tok = args.ref_tokens
    for s in range(args.warmup + args.steps):
        v, det = time_oracle(w, x, n_tok, 1000 + s)
        if s >= args.warmup:
            per_step.append(v)
    value = statistics.median(per_step)
    cores = det["threads"]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": w.B * w.Lq / value * 1e3, "higher_is_better": True, "scaling": "strong",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(w, args.gpus),
        "extrapolated": True,
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "extrapolated": True,
                         "sample": f"per step: stats + selection on the whole {w.name} workload, "
                                   f"masked fp64 attention on {n_tok} random query positions x "
                                   f"{w.Hq} heads; tokens/s = sampled tokens / (their attention "
                                   f"time + stats/selection time pro-rated per token)"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- CUDA arm

def measure_prefill_workload(spa, torch, cid: int, steps: int, warmup: int, peaks: dict,
                             peak_src: str, flush, stream, world: int, rank_max, barrier,
                             device_index: int) -> dict:
    """One prefill workload timed like the headline step (stats -> select ->
    attention, inputs resident, L2 flushed between steps, CUDA events per kernel,
    clocks sampled during the timed region)."""
    w = WORKLOADS[cid]
    x = generate(w)
    if w.dtype == "bf16":
        conv = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
    else:
        conv = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    q, k, v = conv(x["q"]), conv(x["k"]), conv(x["v"])
    del x
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    nb = -(-L // w.block)
    mean = torch.empty((B, Hkv, nb, d), device="cuda", dtype=torch.float32)
    var = torch.empty_like(mean)
    idx = torch.empty((B, Hq, nb, nb), device="cuda", dtype=torch.int32)
    cnt = torch.empty((B, Hq, nb), device="cuda", dtype=torch.int32)
    out = torch.empty_like(q)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        spa.spa_block_stats(k, w.block, mean=mean, var=var)
        if ev:
            ev[1].record(stream)
        spa.spa_select(q, mean, var, L, w.block, w.scale, w.top_p, w.n_sink, w.n_local, w.k_min,
                       idx=idx, count=cnt)
        if ev:
            ev[2].record(stream)
        spa.spa_sparse_attn_prefill(q, k, v, w.block, idx, cnt, w.scale, out=out)
        if ev:
            ev[3].record(stream)

    for _ in range(warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert spa.spa_get_device_error() == 0
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    clocks = ClockSampler(device_index)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    for s_ in range(steps):
        flush.zero_()
        step(evs[s_])
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    total_ms = rank_max(sum(e[0].elapsed_time(e[3]) for e in evs))
    t_att = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    count_h = cnt.cpu().numpy()
    F = kept_flops(count_h, idx.cpu().numpy(), L, w.block, d)
    achieved = F / (t_att / 1e3) / 1e12
    if w.dtype == "bf16":
        bound, peak = "tensor", peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
        psrc = f"{peak_src} bf16_tflops (burst)"
    else:
        # fp32 FFMA on the CUDA cores: 148 SMs x 128 lanes x 2 FLOP per clock
        mhz = peaks.get("sm_max_mhz", 1965.0)
        bound, peak = "alu", 148 * 128 * 2 * mhz * 1e6 / 1e12
        psrc = f"derived: 148 SMs x 128 FP32 lanes x 2 FLOP x {mhz:.0f} MHz"
    res = {"workload": w.name, "tokens/s": job_throughput(B * L, world, steps, total_ms),
           "ms_per_step": total_ms / steps, "steps": steps,
           "block_stats_ms": statistics.mean(e[0].elapsed_time(e[1]) for e in evs),
           "select_ms": statistics.mean(e[1].elapsed_time(e[2]) for e in evs),
           "attn_ms": t_att, "kept_flops_per_launch": F, "TFLOP/s": achieved,
           "bound": bound, "peak": peak, "peak_source": psrc, "frac": achieved / peak,
           "kept_fraction": float(count_h.sum()) / (B * Hq * nb * (nb + 1) / 2),
           "clocks": clk}
    del q, k, v, mean, var, idx, cnt, out
    torch.cuda.empty_cache()
    return res



def prefill_diagnostics(spa, torch, wl, q, k, v) -> dict:
    """Diagnostics of the selection on one prefill workload, from the library's own
    kernels only: the kept fraction of the causal blocks per (b, head, query block)
    (mean, p50, p99), the operator MSE of the sparse output against dense causal
    attention (the same prefill at top_p = 1, which keeps every block), and the
    attention-mass coverage of the kept set per query row, exp(lse_sparse -
    lse_dense): the share of the dense softmax mass that falls on kept keys."""
    sp = spa.prefill(q, k, v, wl.block, wl.top_p, wl.scale, wl.n_sink, wl.n_local, wl.k_min,
                     want_lse=True)
    de = spa.prefill(q, k, v, wl.block, 1.0, wl.scale, wl.n_sink, wl.n_local, wl.k_min,
                     want_lse=True)
    torch.cuda.synchronize()
    nq = sp["count"].shape[-1]
    causal = torch.arange(1, nq + 1, device="cuda", dtype=torch.float32)
    frac = (sp["count"].float() / causal).flatten()
    os_, od = sp["out"].float(), de["out"].float()
    mse = float(((os_ - od) ** 2).mean())
    cov = torch.exp(sp["lse"] - de["lse"]).flatten()
    qs = torch.tensor([0.01, 0.5, 0.99], device="cuda")
    fq = torch.quantile(frac, qs).tolist()
    cq = torch.quantile(cov, qs).tolist()
    return {"kept_fraction": {"mean": float(frac.mean()), "p50": fq[1], "p99": fq[2]},
            "mse_vs_dense": mse, "mse_rel": mse / float((od ** 2).mean()),
            "coverage": {"mean": float(cov.mean()), "p1": cq[0], "p50": cq[1]}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["spa", "reference"], default="spa")
    ap.add_argument("--workload", type=int, default=3)
    ap.add_argument("--decode-workload", type=int, default=5)
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="override the decode workload's batch (smaller captures for profiling)")
    ap.add_argument("--no-rla", action="store_true",
                    help="skip the Residual Linear Attention leg")
    ap.add_argument("--taus", default="0.001,0.002,0.005,0.01,0.02",
                    help="early-stop thresholds swept in the score-ordered traversal leg "
                         "('' to skip)")
    ap.add_argument("--seg-blocks", type=int, default=16,
                    help="segment length (in blocks) of the segmented-permutation leg (0: skip)")
    ap.add_argument("--no-quant", action="store_true",
                    help="skip the selection on quantised statistics in the decode leg")
    ap.add_argument("--no-diagnostics", action="store_true",
                    help="skip the kept-fraction / MSE-vs-dense / coverage diagnostics")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--configs", default="1,2,4",
                    help="other prefill workloads timed beside the headline one ('' to skip)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--cpu-tokens", type=int, default=1536)
    ap.add_argument("--ref-tokens", type=int, default=48)
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist
    import block_sparse_long_stats_b200 as spa

    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))

    def barrier():
        if world > 1:
            dist.barrier()

    def rank_max(v: float) -> float:
        return max_over_ranks(v, world, "cuda")

    peaks, peak_src = load_peaks()
    w_full = WORKLOADS[args.workload]
    # one GPU: the whole workload; N GPUs: each takes a contiguous share of the
    # (b, kv-head) units (whole batch rows, kv-heads with their query heads), so the
    # job processes every token once (strong scaling; no data-path collective)
    u0, u1 = head_shard(w_full.B, w_full.Hkv, world, rank)
    if world > 1 and not (w_full.B == 1 or (u1 - u0) % w_full.Hkv == 0):
        raise SystemExit("head sharding needs whole batch rows or one batch row")
    if w_full.B == 1:
        g0, g1 = u0, u1
        x = generate(w_full, heads=[(0, g) for g in range(g0, g1)])
        G_ = w_full.G
        x = {"q": x["q"][:, g0 * G_:g1 * G_], "k": x["k"][:, g0:g1], "v": x["v"][:, g0:g1]}
        w = w_full.with_(Hq=(g1 - g0) * G_, Hkv=g1 - g0)
    else:
        b0, b1 = u0 // w_full.Hkv, u1 // w_full.Hkv
        x = generate(w_full, heads=[(b, g) for b in range(b0, b1) for g in range(w_full.Hkv)])
        x = {n: a[b0:b1] for n, a in x.items()}
        w = w_full.with_(B=b1 - b0)

    def dev(a):
        if w.dtype == "bf16":
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda().view(torch.bfloat16)
        return torch.from_numpy(a).cuda()

    q, k, v = dev(x["q"]), dev(x["k"]), dev(x["v"])
    B, Hq, L, d = q.shape
    Hkv = k.shape[1]
    nb = -(-L // w.block)
    mean = torch.empty((B, Hkv, nb, d), device="cuda", dtype=torch.float32)
    var = torch.empty_like(mean)
    idx = torch.empty((B, Hq, nb, nb), device="cuda", dtype=torch.int32)
    cnt = torch.empty((B, Hq, nb), device="cuda", dtype=torch.int32)
    out = torch.empty_like(q)
    flush = L2Flush(torch)
    stream = torch.cuda.current_stream()

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        spa.spa_block_stats(k, w.block, mean=mean, var=var)
        if ev:
            ev[1].record(stream)
        spa.spa_select(q, mean, var, L, w.block, w.scale, w.top_p, w.n_sink, w.n_local, w.k_min,
                       idx=idx, count=cnt)
        if ev:
            ev[2].record(stream)
        spa.spa_sparse_attn_prefill(q, k, v, w.block, idx, cnt, w.scale, out=out)
        if ev:
            ev[3].record(stream)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    assert spa.spa_get_device_error() == 0

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    barrier()
    torch.cuda.synchronize()
    for s in range(args.steps):
        flush.zero_()          # L2 flush between timed steps (outside the events)
        step(evs[s])
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    t_stats = [e[0].elapsed_time(e[1]) for e in evs]
    t_sel = [e[1].elapsed_time(e[2]) for e in evs]
    t_att = [e[2].elapsed_time(e[3]) for e in evs]
    t_step = [e[0].elapsed_time(e[3]) for e in evs]
    total_ms = rank_max(sum(t_step))
    ms_per_step = total_ms / args.steps
    # every token of the job once per step (the ranks hold disjoint head shares)
    value = job_throughput(w_full.B * L, 1, args.steps, total_ms)

    count_h = cnt.cpu().numpy()
    idx_h = idx.cpu().numpy()
    F = kept_flops(count_h, idx_h, L, w.block, d)
    att_ms = statistics.mean(t_att)
    achieved = F / (att_ms / 1e3) / 1e12
    # the timed region is well under a second of back-to-back launches: the burst
    # peak is the one to compare with (the sustained one is reported beside it)
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_sus = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    dense_tiles = B * Hq * nb * (nb + 1) / 2
    kept_frac = float(count_h.sum()) / dense_tiles
    stats_bytes = B * Hkv * L * d * 2 + 2 * B * Hkv * nb * d * 4
    per_kernel = {
        "block_stats": {"ms": statistics.mean(t_stats),
                        "GB/s": stats_bytes / (statistics.mean(t_stats) / 1e3) / 1e9},
        # bytes: Q read once to pool it, the statistics once (then L2-resident)
        "select": {"ms": statistics.mean(t_sel),
                   "GB/s": (q.numel() * q.element_size() + 2 * mean.numel() * 4)
                   / (statistics.mean(t_sel) / 1e3) / 1e9,
                   "share_of_step": statistics.mean(t_sel) / (total_ms / args.steps)},
        "sparse_attn_prefill": {"ms": att_ms, "TFLOP/s": achieved},
    }

    # ---- end to end through host buffers: spa_prefill_host copies each chunk of
    # (b, kv-head) pairs in, runs the three kernels on it and copies its output out,
    # pipelined over three streams (inputs pinned, as a serving process keeps them)
    qh, kh, vh = (torch.from_numpy(np.ascontiguousarray(x[n]).view(np.int16))
                  .view(torch.bfloat16).pin_memory() for n in ("q", "k", "v"))
    oh = torch.empty(out.shape, dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(spa.spa_prefill_host_workspace_bytes(torch.bfloat16, B, Hq, Hkv, L, d,
                                                          w.block),
                     dtype=torch.uint8, device="cuda")

    def e2e_step():
        spa.spa_prefill_host(qh, kh, vh, w.block, w.top_p, w.scale, w.n_sink, w.n_local,
                             w.k_min, out=oh, workspace=ws, stream=stream)

    e2e_step()                                   # untimed: creates the pipeline's streams
    e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
             for _ in range(args.e2e_steps)]
    barrier()
    torch.cuda.synchronize()
    for s in range(args.e2e_steps):
        e_evs[s][0].record(stream)
        e2e_step()
        e_evs[s][1].record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = rank_max(sum(a.elapsed_time(b) for a, b in e_evs)) / args.e2e_steps
    e2e = {"value": job_throughput(w_full.B * L, 1, 1, e2e_ms), "unit": "tokens/s",
           "h2d_bytes_per_step": int((qh.numel() + kh.numel() + vh.numel()) * 2) * world,
           "d2h_bytes_per_step": int(oh.numel() * 2) * world, "ms_per_step": e2e_ms,
           "api": "spa_prefill_host (pinned host buffers, copies pipelined with the kernels)"}
    del qh, kh, vh, oh, ws

    # ---- Residual Linear Attention leg (the branch over the blocks the lists leave out)
    rla = None
    # the legs beside the headline step run on one GPU (the scaling run times the step)
    legs = world == 1
    if legs and not args.no_rla:
        states = torch.empty((B, Hkv, nb, d, d), device="cuda", dtype=torch.bfloat16)
        rout = torch.empty((B, Hq, L, d), device="cuda", dtype=torch.float32)
        for _ in range(3):
            spa.spa_rla_block_states(k, v, w.block, states=states)
            spa.spa_rla_prefill(q, k, v, states, w.block, idx, cnt, out=rout)
        torch.cuda.synchronize()
        assert spa.spa_get_device_error() == 0
        n_rla = max(10, args.steps // 2)
        r_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(n_rla)]
        barrier()
        torch.cuda.synchronize()
        for s in range(n_rla):
            flush.zero_()
            r_evs[s][0].record(stream)
            spa.spa_rla_block_states(k, v, w.block, states=states)
            r_evs[s][1].record(stream)
            spa.spa_rla_prefill(q, k, v, states, w.block, idx, cnt, out=rout)
            r_evs[s][2].record(stream)
        torch.cuda.synchronize()
        barrier()
        t_st = rank_max(statistics.mean(e[0].elapsed_time(e[1]) for e in r_evs))
        t_rla = rank_max(statistics.mean(e[1].elapsed_time(e[2]) for e in r_evs))
        # residual blocks before each query block (its own block is always kept here)
        n_res = float(sum(i for i in range(nb)) * B * Hq - (count_h.sum() - B * Hq * nb))
        st_bytes = 2 * k.numel() * 2 + states.numel() * 2
        rla_flops = n_res * 2 * 128 * d * d
        rla = {"states_ms": t_st, "states_GB/s": st_bytes / (t_st / 1e3) / 1e9,
               "states_bytes": st_bytes, "branch_ms": t_rla,
               "residual_blocks": n_res, "branch_flops": rla_flops,
               "branch_TFLOP/s": rla_flops / (t_rla / 1e3) / 1e12,
               "branch_state_bytes_read": n_res * d * d * 2,
               "tokens/s_with_branch": job_throughput(B * L, world, 1,
                                                      ms_per_step + t_st + t_rla)}
        del states, rout

    # ---- score-ordered traversal with early stop (S2O, sections 2-3), block 128:
    # a sweep of tau, each with its processed fraction, attention time and operator
    # MSE against dense causal attention; the headline tau is the largest whose MSE
    # stays within 1.1 x the MSE of the top-p selection alone (the error budget)
    early = None
    taus = [float(t) for t in args.taus.split(",") if t.strip()]
    if legs and taus and w.block == 128 and w.dtype == "bf16":
        oidx = torch.empty_like(idx)
        ocnt = torch.empty_like(cnt)
        proc = torch.empty_like(cnt)
        eout = torch.empty_like(q)
        dense = spa.prefill(q, k, v, w.block, 1.0, w.scale, w.n_sink, w.n_local, w.k_min)["out"]
        torch.cuda.synchronize()
        dense_f = dense.float()
        dense_ms = float(dense_f.pow(2).mean())
        mse_topp = float((out.float() - dense_f).pow(2).mean())
        del dense
        spa.spa_select_score_order(q, mean, var, w.block, w.scale, w.top_p, w.n_sink,
                                   w.n_local, w.k_min, idx=oidx, count=ocnt)
        n_es = max(5, args.steps // 4)
        sweep = []
        for tau in taus:
            for _ in range(3):
                spa.spa_sparse_attn_prefill_early_stop(q, k, v, w.block, oidx, ocnt, w.scale, tau,
                                                       w.n_sink, w.n_local, out=eout,
                                                       processed=proc)
            torch.cuda.synchronize()
            assert spa.spa_get_device_error() == 0
            es_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                      for _ in range(n_es)]
            barrier()
            torch.cuda.synchronize()
            for s_ in range(n_es):
                flush.zero_()
                es_evs[s_][0].record(stream)
                spa.spa_sparse_attn_prefill_early_stop(q, k, v, w.block, oidx, ocnt, w.scale, tau,
                                                       w.n_sink, w.n_local, out=eout,
                                                       processed=proc)
                es_evs[s_][1].record(stream)
            torch.cuda.synchronize()
            barrier()
            t_es = rank_max(statistics.mean(a_.elapsed_time(b_) for a_, b_ in es_evs))
            pr = proc.cpu().numpy()
            oi = oidx.cpu().numpy()
            trunc = np.where(np.arange(oi.shape[-1]) < pr[..., None], oi, -1)
            F_es = kept_flops(pr, np.sort(np.where(trunc < 0, 1 << 30, trunc), axis=-1), L,
                              w.block, d)
            mse = float((eout.float() - dense_f).pow(2).mean())
            sweep.append({"tau": tau,
                          "processed_fraction": float(pr.sum()) / float(count_h.sum()),
                          "attn_ms": t_es, "processed_flops": F_es,
                          "TFLOP/s": F_es / (t_es / 1e3) / 1e12,
                          "mse_vs_dense": mse, "mse_rel": mse / dense_ms,
                          "within_budget": mse <= 1.1 * mse_topp})
        # the selection in traversal order, timed once more on its own
        so_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(n_es)]
        for s_ in range(n_es):
            flush.zero_()
            so_evs[s_][0].record(stream)
            spa.spa_select_score_order(q, mean, var, w.block, w.scale, w.top_p, w.n_sink,
                                       w.n_local, w.k_min, idx=oidx, count=ocnt)
            so_evs[s_][1].record(stream)
        torch.cuda.synchronize()
        t_osel = rank_max(statistics.mean(a_.elapsed_time(b_) for a_, b_ in so_evs))
        ok = [r for r in sweep if r["within_budget"]]
        head = max(ok, key=lambda r: r["tau"]) if ok else None
        early = {"budget": {"mse_top_p_vs_dense": mse_topp, "mse_rel_top_p": mse_topp / dense_ms,
                            "rule": "largest tau with mse_vs_dense <= 1.1 x mse_top_p_vs_dense"},
                 "select_score_order_ms": t_osel, "sweep": sweep,
                 "headline": None if head is None else {
                     "tau": head["tau"], "processed_fraction": head["processed_fraction"],
                     "attn_ms": head["attn_ms"], "TFLOP/s": head["TFLOP/s"],
                     "tokens/s": job_throughput(B * L, world, 1, statistics.mean(t_stats) +
                                                t_osel + head["attn_ms"])}}
        del oidx, ocnt, proc, eout, dense_f

    # ---- segmented key permutation (PBS, sections 2-3)
    pbs = None
    if legs and args.seg_blocks > 0 and w.dtype == "bf16" and args.seg_blocks * w.block <= 8192:
        perm = torch.empty((B, Hkv, L), device="cuda", dtype=torch.int32)
        pws = torch.empty(spa.spa_pbs_workspace_bytes(B, Hq, Hkv, L, w.block), dtype=torch.uint8,
                          device="cuda")
        kp, vp = torch.empty_like(k), torch.empty_like(v)
        mp, vp_ = torch.empty_like(mean), torch.empty_like(var)
        pidx, pcnt = torch.empty_like(idx), torch.empty_like(cnt)
        pout = torch.empty_like(q)

        def pbs_step(ev=None):
            if ev:
                ev[0].record(stream)
            spa.spa_pbs_permutation(q, k, w.block, args.seg_blocks, w.scale, perm=perm,
                                    workspace=pws)
            spa.spa_pbs_gather(k, perm, xp=kp)
            spa.spa_pbs_gather(v, perm, xp=vp)
            spa.spa_block_stats(kp, w.block, mean=mp, var=vp_)
            if ev:
                ev[1].record(stream)
            spa.spa_select_segperm(q, mean, var, mp, vp_, w.block, args.seg_blocks, w.scale,
                                   w.top_p, w.n_sink, w.n_local, w.k_min, idx=pidx, count=pcnt)
            if ev:
                ev[2].record(stream)
            spa.spa_sparse_attn_prefill_segperm(q, k, v, kp, vp, w.block, args.seg_blocks, pidx,
                                                pcnt, w.scale, out=pout)
            if ev:
                ev[3].record(stream)
        for _ in range(3):
            spa.spa_block_stats(k, w.block, mean=mean, var=var)
            pbs_step()
        torch.cuda.synchronize()
        assert spa.spa_get_device_error() == 0
        n_pb = max(5, args.steps // 4)
        pb_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_pb)]
        barrier()
        torch.cuda.synchronize()
        for s_ in range(n_pb):
            flush.zero_()
            pbs_step(pb_evs[s_])
        torch.cuda.synchronize()
        barrier()
        t_perm = rank_max(statistics.mean(e[0].elapsed_time(e[1]) for e in pb_evs))
        t_psel = rank_max(statistics.mean(e[1].elapsed_time(e[2]) for e in pb_evs))
        t_patt = rank_max(statistics.mean(e[2].elapsed_time(e[3]) for e in pb_evs))
        pc = pcnt.cpu().numpy()
        F_p = kept_flops(pc, pidx.cpu().numpy(), L, w.block, d)
        dev_ = (pout.float() - out.float())
        pbs = {"seg_blocks": args.seg_blocks,
               "kept_fraction": float(pc.sum()) / dense_tiles, "kept_fraction_plain": kept_frac,
               "permute_gather_stats_ms": t_perm, "select_ms": t_psel, "attn_ms": t_patt,
               "TFLOP/s": F_p / (t_patt / 1e3) / 1e12,
               "tokens/s": job_throughput(B * L, world, 1, t_perm + t_psel + t_patt +
                                          statistics.mean(t_stats)),
               "vs_plain_output": {"max_abs": float(dev_.abs().max().item()),
                                   "rms": float(dev_.pow(2).mean().sqrt().item())}}
        del perm, pws, kp, vp, mp, vp_, pidx, pcnt, pout

    # ---- decode leg
    decode = None
    if legs and not args.no_decode:
        wd = WORKLOADS[args.decode_workload]
        if args.decode_batch:
            wd = wd.with_(B=args.decode_batch)
        xd = generate(wd)
        qd_ = torch.from_numpy(np.ascontiguousarray(xd["q"]).view(np.int16)).cuda().view(torch.bfloat16)
        kc = torch.from_numpy(np.ascontiguousarray(xd["k"]).view(np.int16)).cuda().view(torch.bfloat16)
        vc = torch.from_numpy(np.ascontiguousarray(xd["v"]).view(np.int16)).cuda().view(torch.bfloat16)
        del xd
        dm, dv = spa.spa_block_stats(kc, wd.block)
        st_ms = []
        for _ in range(5):
            flush.zero_()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            spa.spa_block_stats(kc, wd.block, mean=dm, var=dv)
            e1.record(stream)
            torch.cuda.synchronize()
            st_ms.append(e0.elapsed_time(e1))
        st_bytes = kc.numel() * 2 + 2 * dm.numel() * 4
        stats_full = {"ms": statistics.median(st_ms[1:]),
                      "GB/s": st_bytes / (statistics.median(st_ms[1:]) / 1e3) / 1e9,
                      "bytes": st_bytes}
        didx = torch.empty((wd.B, wd.Hq, 1, wd.nb), device="cuda", dtype=torch.int32)
        dcnt = torch.empty((wd.B, wd.Hq, 1), device="cuda", dtype=torch.int32)
        ws = torch.empty(spa.spa_decode_workspace_bytes(wd.B, wd.Hq, wd.Hkv, wd.T, wd.d, wd.block),
                         dtype=torch.uint8, device="cuda")
        dout = torch.empty_like(qd_)
        for _ in range(3):
            spa.spa_select(qd_, dm, dv, wd.T, wd.block, wd.scale, wd.top_p, idx=didx, count=dcnt)
            spa.spa_sparse_attn_decode(qd_, kc, vc, wd.block, didx, dcnt, wd.scale, workspace=ws,
                                       out=dout)
        torch.cuda.synchronize()
        assert spa.spa_get_device_error() == 0
        n_dec = max(10, args.steps // 2)
        last = wd.nb - 1      # the block the new token lands in: its statistics are updated
        # a decode step: statistics of the newest block, selection, attention
        d_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_dec)]
        barrier()
        torch.cuda.synchronize()
        for s in range(n_dec):
            flush.zero_()
            d_evs[s][0].record(stream)
            spa.spa_block_stats(kc, wd.block, last, last + 1, mean=dm, var=dv)
            d_evs[s][1].record(stream)
            spa.spa_select(qd_, dm, dv, wd.T, wd.block, wd.scale, wd.top_p, idx=didx, count=dcnt)
            d_evs[s][2].record(stream)
            spa.spa_sparse_attn_decode(qd_, kc, vc, wd.block, didx, dcnt, wd.scale, workspace=ws,
                                       out=dout)
            d_evs[s][3].record(stream)
        torch.cuda.synchronize()
        barrier()
        t_dupd = rank_max(statistics.mean(e[0].elapsed_time(e[1]) for e in d_evs))
        t_dsel = rank_max(statistics.mean(e[1].elapsed_time(e[2]) for e in d_evs))
        t_dec = rank_max(statistics.mean(e[2].elapsed_time(e[3]) for e in d_evs))
        dbytes = kept_kv_bytes(dcnt.cpu().numpy(), didx.cpu().numpy(), wd.G, wd.T, wd.block, wd.d)
        gbs = dbytes / (t_dec / 1e3) / 1e9
        drla = None
        if not args.no_rla:
            dstate = torch.zeros((wd.B, wd.Hkv, wd.d, wd.d), device="cuda", dtype=torch.float32)
            ws_r = torch.empty(spa.spa_rla_decode_workspace_bytes(wd.B, wd.Hq, wd.Hkv, wd.T, wd.d,
                                                                  wd.block),
                               dtype=torch.uint8, device="cuda")
            orla = torch.empty(qd_.shape, device="cuda", dtype=torch.float32)
            sb_ms = []
            for _ in range(4):
                flush.zero_()
                dstate.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                spa.spa_rla_decode_state(kc, vc, state=dstate)
                e1.record(stream)
                torch.cuda.synchronize()
                sb_ms.append(e0.elapsed_time(e1))
            for _ in range(3):
                spa.spa_sparse_attn_decode_rla(qd_, kc, vc, dstate, wd.block, didx, dcnt, wd.scale,
                                               workspace=ws_r, out=dout, out_rla=orla)
            torch.cuda.synchronize()
            assert spa.spa_get_device_error() == 0
            r_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                     for _ in range(n_dec)]
            barrier()
            torch.cuda.synchronize()
            for s in range(n_dec):
                flush.zero_()
                r_evs[s][0].record(stream)
                spa.spa_sparse_attn_decode_rla(qd_, kc, vc, dstate, wd.block, didx, dcnt, wd.scale,
                                               workspace=ws_r, out=dout, out_rla=orla)
                r_evs[s][1].record(stream)
            torch.cuda.synchronize()
            barrier()
            t_drla = rank_max(statistics.mean(a_.elapsed_time(b_) for a_, b_ in r_evs))
            sb = statistics.median(sb_ms[1:])
            drla = {"state_build_ms": sb,
                    "state_build_GB/s": 2 * kc.numel() * 2 / (sb / 1e3) / 1e9,
                    "attn_with_branch_ms": t_drla,
                    "GB/s": (dbytes + dstate.numel() * 4) / (t_drla / 1e3) / 1e9,
                    "tokens/s": world * wd.B / ((t_dsel + t_drla) / 1e3)}
            del dstate, ws_r, orla
        # selection on INT4 or FP4 microscale statistics (SpotAttention, section 4)
        def quant_step(fmt):
            qrec = spa.spa_quantize_block_stats(dm, dv, wd.T, wd.block, fmt=fmt)
            qi = torch.empty_like(didx)
            qc = torch.empty_like(dcnt)
            q_ms = []
            for _ in range(4):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                spa.spa_quantize_block_stats(dm, dv, wd.T, wd.block, qstats=qrec, fmt=fmt)
                e1.record(stream)
                torch.cuda.synchronize()
                q_ms.append(e0.elapsed_time(e1))
            for _ in range(3):
                spa.spa_select_quantized(qd_, qrec, wd.T, wd.block, wd.scale, wd.top_p, idx=qi,
                                         count=qc, fmt=fmt)
            torch.cuda.synchronize()
            assert spa.spa_get_device_error() == 0
            # the decode step on records: statistics and record of the newest block in
            # one kernel, selection on the records, attention on its lists
            qs_evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(n_dec)]
            qout = torch.empty_like(dout)
            for _ in range(3):
                spa.spa_block_stats_quantized(kc, wd.block, last, last + 1, dm, dv, qrec, fmt=fmt)
                spa.spa_select_quantized(qd_, qrec, wd.T, wd.block, wd.scale, wd.top_p, idx=qi,
                                         count=qc, fmt=fmt)
                spa.spa_sparse_attn_decode(qd_, kc, vc, wd.block, qi, qc, wd.scale, workspace=ws,
                                           out=qout)
            torch.cuda.synchronize()
            assert spa.spa_get_device_error() == 0
            barrier()
            torch.cuda.synchronize()
            for s in range(n_dec):
                flush.zero_()
                qs_evs[s][0].record(stream)
                spa.spa_block_stats_quantized(kc, wd.block, last, last + 1, dm, dv, qrec, fmt=fmt)
                qs_evs[s][1].record(stream)
                spa.spa_select_quantized(qd_, qrec, wd.T, wd.block, wd.scale, wd.top_p, idx=qi,
                                         count=qc, fmt=fmt)
                qs_evs[s][2].record(stream)
                spa.spa_sparse_attn_decode(qd_, kc, vc, wd.block, qi, qc, wd.scale, workspace=ws,
                                           out=qout)
                qs_evs[s][3].record(stream)
            torch.cuda.synchronize()
            barrier()
            t_qupd = rank_max(statistics.mean(e[0].elapsed_time(e[1]) for e in qs_evs))
            t_qsel = rank_max(statistics.mean(e[1].elapsed_time(e[2]) for e in qs_evs))
            t_qdec = rank_max(statistics.mean(e[2].elapsed_time(e[3]) for e in qs_evs))
            qbytes = kept_kv_bytes(qc.cpu().numpy(), qi.cpu().numpy(), wd.G, wd.T, wd.block, wd.d)
            res = {"format": fmt, "stats_bytes_fp32": 2 * dm.numel() * 4, "stats_bytes_records": qrec.numel(),
                  "quantize_full_cache_ms": statistics.median(q_ms[1:]),
                  "update_newest_block_ms": t_qupd, "select_ms": t_qsel, "attn_ms": t_qdec,
                  "kept_kv_bytes": qbytes, "GB/s": qbytes / (t_qdec / 1e3) / 1e9,
                  "kept_fraction": float(qc.float().mean().item()) / wd.nb,
                  "tokens/s": world * wd.B / ((t_qupd + t_qsel + t_qdec) / 1e3)}
            del qout
            del qrec, qi, qc
            return res

        dq = None
        if not args.no_quant:
            dq = quant_step("int4")
            dq["fp4"] = quant_step("fp4")
        decode = {"workload": wd.name, "kept_kv_bytes": dbytes, "attn_ms": t_dec,
                  "update_newest_block_ms": t_dupd, "select_ms": t_dsel,
                  "select_GB/s": 2 * dm.numel() * 4 / (t_dsel / 1e3) / 1e9,
                  "select_share_of_step": t_dsel / (t_dupd + t_dsel + t_dec),
                  "GB/s": gbs, "peak_GB/s": peaks["hbm_gbs"],
                  "frac": gbs / peaks["hbm_gbs"], "peak_source": peak_src,
                  "tokens/s": world * wd.B / ((t_dupd + t_dsel + t_dec) / 1e3),
                  "step": "statistics of the newest block, selection on fp32 statistics, "
                          "attention; the step on INT4 records is quantized_stats",
                  "kept_fraction": float(dcnt.float().mean().item()) / wd.nb,
                  "kept_fraction_union": dbytes / float(2 * kc.numel() * kc.element_size()),
                  "block_stats_full_cache": stats_full, "rla": drla, "quantized_stats": dq}
        del kc, vc

    # ---- the other prefill workloads, each timed like the headline step
    configs = {}
    for cid in ([int(c) for c in args.configs.split(",") if c.strip()] if legs else []):
        if cid == args.workload or WORKLOADS[cid].mode != "prefill":
            continue
        n_st = {1: max(args.steps, 20), 4: min(args.steps, 8)}.get(cid, args.steps)
        configs[WORKLOADS[cid].name] = measure_prefill_workload(
            spa, torch, cid, n_st, 3, peaks, peak_src, flush, stream, world, rank_max, barrier,
            local)

    # ---- selection diagnostics on the three prefill workloads (dense comparisons
    # on the 1K, 8K and 32K workloads only; the 128K one would need 140 TFLOP more)
    diag = None
    if legs and not args.no_diagnostics:
        diag = {}
        for cid in (1, 2, args.workload):
            wl = WORKLOADS[cid]
            if wl.mode != "prefill":
                continue
            if cid == args.workload:
                dq, dk, dv = q, k, v
            else:
                xl = generate(wl)
                conv = ((lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16))
                         .cuda().view(torch.bfloat16)) if wl.dtype == "bf16"
                        else (lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()))
                dq, dk, dv = conv(xl["q"]), conv(xl["k"]), conv(xl["v"])
            diag[wl.name] = prefill_diagnostics(spa, torch, wl, dq, dk, dv)
            del dq, dk, dv
        torch.cuda.empty_cache()
        assert spa.spa_get_device_error() == 0

    # ---- CPU oracle baseline (rank 0, one GPU)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        v_cpu, det = time_oracle(w, x, args.cpu_tokens, 7)
        cpu = {"value": v_cpu, "unit": "tokens/s", "cores": det["threads"], "kind": "oracle",
               "extrapolated": True,
               "sample": f"stats + selection on the whole workload ({det['t_select_s']:.2f} s), "
                         f"masked fp64 attention on {args.cpu_tokens} random query positions x "
                         f"{Hq} heads ({det['t_attention_sample_s']:.2f} s); tokens/s = sampled "
                         f"tokens / (their attention time + stats/selection pro-rated per token)"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": workload_config(w_full, world),
            "kept_fraction": kept_frac,
            "roofline": {"bound": "tensor", "kernel": "sparse_attn_prefill", "achieved": achieved,
                         "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                         "peak_source": f"{peak_src} bf16_tflops (burst: the timed region "
                                        f"is {total_ms / 1e3:.2f} s)",
                         "sm_mhz_median": clk.get("sm_mhz"),
                         "peak_sustained": peak_sus, "frac_vs_sustained": achieved / peak_sus,
                         "kept_flops_per_launch": F,
                         "traffic": captured_traffic("prefill_tc_kernel<128>", w.name),
                         "traffic_unit": "bytes per launch (ncu dram read + write)",
                         "algorithmic_bytes": float(2 * q.numel() * 2 + 2 * k.numel() * 2)},
            "kernels": per_kernel,
            "configs": configs,
            "rla": rla,
            "early_stop": early,
            "segmented_permutation": pbs,
            "decode": decode,
            "diagnostics": diag,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "clocks": clk,
            "gpu_launches": 3 * args.steps,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()

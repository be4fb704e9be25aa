#!/usr/bin/env python
"""Benchmark: SATA prefill tokens/s (headline) and decode tokens/s on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sata|reference]

One "step" is one causal SATA prefill of the d_K = d_V = 64, P = 4 workload
(B=1, H=8, N=65536: 47905 features per head) through the C ABI, inputs resident
in HBM.  Decode is measured beside it on the decode workload (B=64, H=32,
d_K = d_V = 32, a state built by an 8192-token prefill, then decode steps) and
reported under "decode", and the backward pass of the prefill (gradients of q,
k, v on the d = 64, P = 4 head shape over 4096 tokens) under "backward".  For N > 1
(torchrun) the job has 8N heads and rank r owns heads [8r, 8r + 8) of it, each
head its own seeded draw (weak scaling: the work per GPU is fixed; no
collective on the data path); times are max over ranks.

--impl reference times the float64 CPU oracle on a bounded sample of the same
workload (the only other code in this file that may run the oracle is the
cpu_baseline leg).
"""
from __future__ import annotations

import argparse
import hashlib
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

METRIC = "SATA prefill tokens/s and decode tokens/s at d_K=64,P=4; % of roofline"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP32_LANES_PER_SM = 128      # fp32 FMA lanes per SM
NUM_SMS = 148


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["sata", "reference"], default="sata")
    ap.add_argument("--workload", default="prefill_d64")
    ap.add_argument("--decode-workload", default="decode_d32")
    ap.add_argument("--decode-steps", type=int, default=None, help="default: all of the workload's")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--backward-workload", default="backward_d64")
    ap.add_argument("--no-backward", action="store_true")
    ap.add_argument("--only", choices=["all", "prefill", "decode", "backward"], default="all",
                    help="run one part only (reduced workloads for profiler captures)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the other prefill workloads")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--path", choices=["auto", "cuda_core", "tensor_core"], default="auto")
    ap.add_argument("--seq-split", action="store_true",
                    help="split each sequence across the ranks (segment states, all-gather, prefix, "
                         "prefill from the prefix): strong scaling of one prefill; the default shards "
                         "heads (weak scaling, no collective)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# --------------------------------------------------------------- helpers ----

class ClockSampler:
    """nvidia-smi samples (200 ms) of SM clock and throttle reasons while running."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id = gpu_id
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.gpu_id, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.th = threading.Thread(target=self._read, daemon=True)
            self.th.start()
        except OSError:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.th.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, val in zip(names, parts[4:8]):
                if val.lower() in ("active", "1"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"], "samples": 0}
        hi = [s for s in sm if s > 0.5 * max(sm)]
        return {"sm_mhz": statistics.median(hi), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def gpu_uuid(torch, dev):
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(dev)


def kernel_source_hash(names):
    """sha256 (16 hex digits) of the kernel's source file(s) under csrc/, in order."""
    h = hashlib.sha256()
    for name in ([names] if isinstance(names, str) else names):
        p = os.path.join(ROOT, "symmetric_taylor_self_b200", "csrc", name)
        if not os.path.exists(p):
            return None
        h.update(open(p, "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's sources
    are unchanged since the capture; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e:
        return None
    if e.get("source_sha256_16") != kernel_source_hash(e.get("source", "")):
        return None
    return e.get("dram_bytes_per_launch")


def flops_per_token(d_K, d_V, P):
    """Algorithmic FLOPs per token per head, the closed form of the page "Self-
    attention at constant cost per token via symmetry-aware Taylor approximation",
    section "Hidden-state size and FLOPs": (4 d_V + 2(P d_K + 1)/(d_K + 1) + 2) F."""
    F = math.comb(d_K + P - 1, P - 1)
    num = (4 * d_V + 2) * (d_K + 1) + 2 * (P * d_K + 1)
    return num * F // (d_K + 1)


# prefill workloads measured beside the headline one (lines under "extra")
EXTRA_WORKLOADS = ("tiny_d8", "prefill_d16", "prefill_d32", "prefill_d128", "prefill_d64_dv32", "prefill_d16_p6")
F32_INPUT_WORKLOADS = ("tiny_d8",)   # specified with fp32 q, k, v


# ---------------------------------------------------------- distributed ----

def dist_setup(torch):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(torch, world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(torch, world, x: float) -> float:
    """Largest x over all ranks (the job's time is the slowest rank's)."""
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step: float, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's units over the slowest rank's time."""
    return units_per_rank_step * steps * world / (max_ms / 1000.0)


def timed(torch, world, fn, K, W, stream):
    for _ in range(W):
        fn()
    torch.cuda.synchronize()
    barrier(torch, world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        fn()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier(torch, world)
    torch.cuda.synchronize()
    return max_over_ranks(torch, world, e0.elapsed_time(e1))


# ------------------------------------------------------------ CPU oracle ----

def cpu_oracle_rate(w, seconds, threads=None):
    """Oracle tokens/s on a bounded sample: `threads` heads of the workload, each
    run from its first token; the token count is calibrated to ~`seconds`."""
    import oracle
    from symmetric_taylor_self_b200 import workloads as wl

    threads = threads or len(os.sched_getaffinity(0))
    heads = [(b, h) for b in range(w.B) for h in range(w.H)][:threads]
    if len(heads) < threads:          # fewer heads than cores: reuse heads
        heads = (heads * ((threads + len(heads) - 1) // len(heads)))[:threads]
    data = {}
    for bh in set(heads):
        q, k, v = wl.head_inputs(w, *bh)
        data[bh] = (q, k, v)
    from concurrent.futures import ThreadPoolExecutor

    def run(T):
        def one(bh):
            q, k, v = data[bh]
            oracle.scan(q[:T], k[:T], v[:T], w.P)
        t0 = time.perf_counter()
        with ThreadPoolExecutor(max_workers=len(heads)) as ex:
            list(ex.map(one, heads))
        return time.perf_counter() - t0

    T0 = 16
    dt = run(T0)
    T = int(max(T0, min(w.N, T0 * seconds / max(dt, 1e-3))))
    dt = run(T)
    return {"value": len(heads) * T / dt, "unit": "tokens/s", "cores": len(heads), "kind": "oracle",
            "sample": f"{len(heads)} heads x first {T} tokens of {w.name} (float64 C recurrence, one thread per head)",
            "seconds": dt}


# ----------------------------------------------------------------- main ----

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    from symmetric_taylor_self_b200 import workloads as wl
    w = wl.WORKLOADS[args.workload]
    per_step = max(1.0, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_rate(w, per_step / 4)
    vals, secs = [], 0.0
    for _ in range(args.steps):
        r = cpu_oracle_rate(w, per_step)
        vals.append(r["value"])
        secs += r["seconds"]
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * secs / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d_K={w.d_K} d_V={w.d_V} P={w.P}",
                   "sample": r["sample"]},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": r["cores"], "kind": "oracle",
                         "sample": r["sample"]},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)

    import torch

    import symmetric_taylor_self_b200 as sata
    from symmetric_taylor_self_b200 import workloads as wl

    rank, world, local = dist_setup(torch)
    if args.only != "all":
        return run_part(torch, sata, wl, args, world)
    if args.seq_split:
        return run_seq_split(torch, sata, wl, args, rank, world)
    dev = torch.device("cuda", torch.cuda.current_device())
    sata.load()
    sata.sata_set_option(sata.SATA_OPT_PREFILL_PATH, {"auto": 0, "cuda_core": 1, "tensor_core": 2}[args.path])
    peaks, peaks_src = load_peaks()
    stream = torch.cuda.Stream()
    w = wl.WORKLOADS[args.workload]

    # ---------------- prefill (headline) ----------------
    # N ranks: one job of B x (H N) heads, rank r owning heads [H r, H (r + 1)) of every
    # batch row (each its own seeded draw); no collective on the data path
    (q, k, v), _ = wl.make_inputs(w, h0=rank * w.H, H_total=w.H * world)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty((w.B, w.H, w.N, w.d_V), dtype=torch.float32, device=dev)
    in_bytes = sum(t.numel() * t.element_size() for t in (q, k, v))
    out_bytes = out.numel() * 4

    def step():
        sata.sata_prefill_ex(qd, kd, vd, out, w.B, w.H, w.N, w.d_K, w.d_V, w.P, None, None, stream)

    with torch.cuda.stream(stream):
        step()                                   # allocates the library workspace
    torch.cuda.synchronize()
    if sata.sata_sync_status(stream) != 0:
        raise RuntimeError("device status after the first prefill")

    sampler = ClockSampler(gpu_uuid(torch, dev))
    sata.sata_reset_kernel_stats()
    sata.sata_set_option(sata.SATA_OPT_TIME_KERNELS, 1)
    # warm-up first (untimed), then the timed region with per-kernel events
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sata.sata_reset_kernel_stats()
    sampler.start()
    ms = timed(torch, world, step, args.steps, 0, stream)
    clocks = sampler.stop()
    stats = sata.sata_kernel_stats()
    sata.sata_set_option(sata.SATA_OPT_TIME_KERNELS, 0)
    if sata.sata_sync_status(stream) != 0:
        raise RuntimeError("device status after the timed prefill")
    tokens_per_step = w.B * w.N
    value = job_throughput(tokens_per_step, args.steps, world, ms)
    launches = sum(n for n, _ in stats.values())

    roof = prefill_roofline(stats, w, args.steps, peaks, peaks_src, clocks)
    dom = roof["kernel"] if roof else None

    # ---------------- e2e through host buffers ----------------
    e2e = None
    if not args.no_e2e:
        qh, kh, vh = q.pin_memory(), k.pin_memory(), v.pin_memory()
        outh = torch.empty(out.shape, dtype=torch.float32).pin_memory()

        def e2e_step():
            # the public host-buffer entry point: it copies the inputs in and the output out
            # itself, token segment by segment, overlapped with the kernels
            sata.sata_prefill_host(qh, kh, vh, outh, w.B, w.H, w.N, w.d_K, w.d_V, w.P, None, stream)

        ms_e2e = timed(torch, world, e2e_step, args.steps, 1, stream)
        e2e = {"value": job_throughput(tokens_per_step, args.steps, world, ms_e2e), "unit": "tokens/s",
               "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": out_bytes,
               "ms_per_step": ms_e2e / args.steps}

    # ---------------- decode ----------------
    dec = None
    if not args.no_decode:
        dec = bench_decode(torch, sata, wl, args, world, dev, stream, peaks, peaks_src)

    # ---------------- backward of the prefill ----------------
    bwd = None
    if not args.no_backward:
        bwd = bench_backward(torch, sata, wl, args, world, dev, stream, peaks, peaks_src)

    # ---------------- the other prefill workloads ----------------
    extra = []
    for name in ([] if args.no_extra else EXTRA_WORKLOADS):
        e = bench_extra(torch, sata, wl, name, args, world, dev, stream, peaks, peaks_src)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            e["cpu_baseline"] = cpu_oracle_rate(wl.WORKLOADS[name], min(args.cpu_seconds, 4.0))
        extra.append(e)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16" if dom and dom.startswith("tc") else "f32",
        "accumulate": "f32", "data": "synthetic (seeded N(0,1) bf16 inputs; no dataset involved)",
        "config": {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d_K={w.d_K} d_V={w.d_V} P={w.P} "
                               f"F={w.F}", "per_rank_batch": w.B, "seq_len": w.N,
                   "parallelism": (f"heads sharded: rank r owns heads [{w.H}r, {w.H}(r+1)) of a "
                                   f"{w.H * world}-head job, no collective") if world > 1 else "one GPU",
                   "l2": f"inputs {in_bytes / 1e6:.0f} MB + output {out_bytes / 1e6:.0f} MB per step > 126 MB L2",
                   "path": args.path},
        "roofline": roof, "gpu_launches": launches, "clocks": clocks, "e2e": e2e, "decode": dec,
        "backward": bwd, "extra": extra,
        "kernel_ms": {k_: {"launches": n, "ms": t} for k_, (n, t) in stats.items()},
        "peaks_source": peaks_src,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_oracle_rate(w, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def prefill_roofline(stats, w, steps, peaks, peaks_src, clocks):
    """Roofline of the prefill's dominant kernel: algorithmic FLOPs of the
    workload per launch over its mean CUDA-event duration."""
    if not stats:
        return None
    dom = max(stats, key=lambda n: stats[n][1])
    n_l, ms_l = stats[dom]
    per_launch_ms = ms_l / n_l
    flops_per_launch = flops_per_token(w.d_K, w.d_V, w.P) * w.B * w.H * w.N * steps / n_l
    achieved = flops_per_launch / (per_launch_ms / 1000.0) / 1e12
    if dom.startswith("tc"):
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "peak_kind": f"{peaks_src} bf16 dense burst (fp16 operands run at the bf16 rate)"}
    else:
        sm_ghz = ((clocks or {}).get("sm_max_mhz") or 1965.0) / 1000.0
        alu_peak = NUM_SMS * FP32_LANES_PER_SM * 2 * sm_ghz / 1000.0
        roof = {"bound": "alu", "achieved": achieved, "peak": alu_peak, "unit": "TFLOP/s",
                "peak_kind": "fp32 FMA: 148 SMs x 128 lanes x 2 FLOP x max SM clock"}
    roof["frac"] = roof["achieved"] / roof["peak"]
    roof["kernel"] = dom
    roof["launches_per_step"] = n_l / steps
    roof["ms_per_launch"] = per_launch_ms
    roof["algorithmic_flops_per_launch"] = flops_per_launch
    tr = ncu_traffic(dom)
    roof["traffic"] = tr
    if tr is None:
        roof["traffic_note"] = "no ncu capture of the current kernel source"
    return roof


def bench_extra(torch, sata, wl, name, args, world, dev, stream, peaks, peaks_src):
    """One more prefill workload, each timed step preceded (outside its events)
    by a 256 MB write that flushes L2, since some of these inputs fit in L2.  The
    workloads specified with fp32 inputs (tiny_d8) run on them as drawn
    (sata_prefill_f32); the others take the bf16 inputs."""
    w = wl.WORKLOADS[name]
    f32_in = name in F32_INPUT_WORKLOADS
    (q, k, v), _ = wl.make_inputs(w, dtype=torch.float32 if f32_in else torch.bfloat16)
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.empty((w.B, w.H, w.N, w.d_V), dtype=torch.float32, device=dev)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)

    def step():
        if f32_in:
            sata.sata_prefill_f32(qd, kd, vd, out, w.B, w.H, w.N, w.d_K, w.d_V, w.P, None, stream)
        else:
            sata.sata_prefill_ex(qd, kd, vd, out, w.B, w.H, w.N, w.d_K, w.d_V, w.P, None, None, stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    sata.sata_reset_kernel_stats()
    sata.sata_set_option(sata.SATA_OPT_TIME_KERNELS, 1)
    total = 0.0
    for _ in range(args.steps):
        with torch.cuda.stream(stream):
            flush.fill_(1.0)
        total += timed(torch, world, step, 1, 0, stream)
    stats = sata.sata_kernel_stats()
    sata.sata_set_option(sata.SATA_OPT_TIME_KERNELS, 0)
    if sata.sata_sync_status(stream) != 0:
        raise RuntimeError(f"device status after {name}")
    roof = prefill_roofline(stats, w, args.steps, peaks, peaks_src, None)
    line = {"metric": "SATA prefill tokens/s", "workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d_K={w.d_K} "
            f"d_V={w.d_V} P={w.P} F={w.F}", "value": job_throughput(w.B * w.N, args.steps, world, total),
            "unit": "tokens/s", "steps": args.steps, "ms_per_step": total / args.steps,
            "inputs": "fp32 q, k, v as drawn" if f32_in else "bf16 q, k, v",
            "dtype": "f16" if roof and roof["kernel"].startswith("tc") else "f32",
            "l2": "L2 flushed (256 MB write) before each timed step", "roofline": roof,
            "gpu_launches": sum(n for n, _ in stats.values()),
            "kernel_ms": {k_: {"launches": n, "ms": t} for k_, (n, t) in stats.items()}}
    del qd, kd, vd, out, flush
    return line


def run_seq_split(torch, sata, wl, args, rank, world):
    """One prefill of the workload's sequences split by token ranges across the
    ranks (seqsplit.py): strong scaling, one JSON line from rank 0."""
    from symmetric_taylor_self_b200 import seqsplit
    dev = torch.device("cuda", torch.cuda.current_device())
    sata.load()
    w = wl.WORKLOADS[args.workload]
    n = -(-w.N // world)
    a, b = min(rank * n, w.N), min((rank + 1) * n, w.N)
    (q, k, v), _ = wl.make_inputs(w)
    qd, kd, vd = (x[:, :, a:b].contiguous().to(dev) for x in (q, k, v))
    stream = torch.cuda.Stream()

    def step():
        with torch.cuda.stream(stream):
            seqsplit.prefill_sequence_split(qd, kd, vd, w.P)

    step()
    torch.cuda.synchronize()
    sampler = ClockSampler(gpu_uuid(torch, dev))
    sampler.start()
    ms = timed(torch, world, step, args.steps, args.warmup, stream)
    clocks = sampler.stop()
    if sata.sata_sync_status(stream) != 0:
        raise RuntimeError("device status after the split prefill")
    value = w.B * w.N * args.steps / (ms / 1000.0)
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None, "dtype": "f16", "accumulate": "f32",
            "data": "synthetic (seeded N(0,1) bf16 inputs; no dataset involved)",
            "config": {"workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d_K={w.d_K} d_V={w.d_V} P={w.P}",
                       "parallelism": f"sequence split over {world} ranks: {n} tokens per rank, segment "
                                      f"states all-gathered, exclusive prefix, prefill from the prefix",
                       "l2": "inputs and state exchange larger than L2 at this size"},
            "roofline": None, "e2e": None, "clocks": clocks,
            "note": "two prefills of each rank's segment plus the state all-gather"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_part(torch, sata, wl, args, world):
    """One part alone, no JSON line: the command profiler captures run."""
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.Stream()
    if args.only == "backward":
        w = wl.WORKLOADS[args.backward_workload]
        (q, k, v), _ = wl.make_inputs(w)
        qd, kd, vd, dy = q.to(dev), k.to(dev), v.to(dev), wl.cotangent(w).to(dev)
        g = [torch.empty(x.shape, dtype=torch.float32, device=dev) for x in (q, k, v)]
        for _ in range(args.warmup + args.steps):
            sata.sata_prefill_backward(qd, kd, vd, dy, *g, w.B, w.H, w.N, w.d_K, w.d_V, w.P, None, stream)
    elif args.only == "prefill":
        w = wl.WORKLOADS[args.workload]
        (q, k, v), _ = wl.make_inputs(w)
        qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
        out = torch.empty((w.B, w.H, w.N, w.d_V), dtype=torch.float32, device=dev)
        for _ in range(args.warmup + args.steps):
            sata.sata_prefill_ex(qd, kd, vd, out, w.B, w.H, w.N, w.d_K, w.d_V, w.P, None, None, stream)
    else:
        w = wl.WORKLOADS[args.decode_workload]
        (q, k, v), (qs, ks, vs) = wl.make_inputs(w)
        st = sata.State(w.B, w.H, w.d_K, w.d_V, w.P, device=dev, stream=stream)
        with torch.cuda.stream(stream):
            sata.prefill(q.to(dev), k.to(dev), v.to(dev), P=w.P, state=st, stream=stream)
        qs, ks, vs = qs.to(dev), ks.to(dev), vs.to(dev)
        for i in range(min(args.warmup + args.steps, w.steps)):
            sata.decode_step(st, qs[i], ks[i], vs[i])
    torch.cuda.synchronize()
    status = sata.sata_sync_status(stream)
    print(json.dumps({"part": args.only, "status": status}), flush=True)
    return 0 if status == 0 else 1


def backward_flops(d_K, d_V, P):
    """Algorithmic FLOPs per token and head of the backward's gradient scans (the
    feature-form contractions; the features, the pairs inside a chunk and the
    recomputed forward not counted).
    Tensor-core path: dq and dk each update and read a state of F2 x d_K x (d_V + 1)
    values, F2 = binom(d_K + P - 2, P - 2) the features of T_{P-1}: 2 x 2 F2 d_K (d_V + 1)
    each; dv is the prefill's scan on the reversed sequence (flops_per_token).
    CUDA-core path: dq scan: S r_t and the S update, 2 x 2F(d_V+1); dk/dv scan: G u_s,
    the dv readout 2F d_V, the G update: 4F(d_V+1) + 2F d_V."""
    F = math.comb(d_K + P - 1, P - 1)
    F2 = math.comb(d_K + P - 2, P - 2) if P >= 2 else 0
    return {"bwd_tc_scan": 8 * F2 * d_K * (d_V + 1) + flops_per_token(d_K, d_V, P),
            "bwd_q_scan": 4 * F * (d_V + 1), "bwd_kv_scan": 4 * F * (d_V + 1) + 2 * F * d_V}


def bench_backward(torch, sata, wl, args, world, dev, stream, peaks, peaks_src):
    """The backward workload; each timed step is preceded (outside its events) by a
    256 MB write that flushes L2, since the step's working set is close to its size."""
    w = wl.WORKLOADS[args.backward_workload]
    (q, k, v), _ = wl.make_inputs(w)
    qd, kd, vd, dy = q.to(dev), k.to(dev), v.to(dev), wl.cotangent(w).to(dev)
    dq = torch.empty((w.B, w.H, w.N, w.d_K), dtype=torch.float32, device=dev)
    dk = torch.empty_like(dq)
    dv = torch.empty((w.B, w.H, w.N, w.d_V), dtype=torch.float32, device=dev)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev)

    def step():
        sata.sata_prefill_backward(qd, kd, vd, dy, dq, dk, dv, w.B, w.H, w.N, w.d_K, w.d_V, w.P, None,
                                   stream)

    with torch.cuda.stream(stream):
        step()                                   # allocates the library workspace
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    sata.sata_reset_kernel_stats()
    sata.sata_set_option(sata.SATA_OPT_TIME_KERNELS, 1)
    ms = 0.0
    for _ in range(args.steps):
        with torch.cuda.stream(stream):
            flush.fill_(1.0)
        ms += timed(torch, world, step, 1, 0, stream)
    stats = sata.sata_kernel_stats()
    sata.sata_set_option(sata.SATA_OPT_TIME_KERNELS, 0)
    if sata.sata_sync_status(stream) != 0:
        raise RuntimeError("device status after the backward")
    value = job_throughput(w.B * w.N, args.steps, world, ms)
    per_tok = backward_flops(w.d_K, w.d_V, w.P)
    roof = None
    scans = {k_: stats[k_] for k_ in per_tok if k_ in stats}
    if "bwd_tc_scan" in scans:
        # three launches a step (dq, dk, dv) of different sizes: the step's scan FLOPs over
        # the step's scan time, i.e. the mean over the three
        n_l, ms_l = scans["bwd_tc_scan"]
        flops_per_launch = per_tok["bwd_tc_scan"] * w.B * w.H * w.N * args.steps / n_l
        achieved = flops_per_launch / (ms_l / n_l / 1000.0) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "kernel": "bwd_tc_scan",
                "launches_per_step": n_l / args.steps, "ms_per_launch": ms_l / n_l,
                "algorithmic_flops_per_launch": flops_per_launch,
                "peak_kind": f"{peaks_src} bf16 dense burst (fp16 operands run at the bf16 rate); FLOPs and "
                             "time are the mean over the step's dq, dk and dv scans",
                "traffic": ncu_traffic("bwd_tc_scan")}
    elif scans:
        # the CUDA-core gradient scans' contractions run on tensor cores with tf32 operands:
        # the tf32 dense peak is the measured bf16 peak times the nominal ratio 1.1 / 2.25
        tf32_peak = peaks["bf16_tflops"] * 1.1 / 2.25
        dom = max(scans, key=lambda n: scans[n][1])
        n_l, ms_l = scans[dom]
        flops_per_launch = per_tok[dom] * w.B * w.H * w.N * args.steps / n_l
        achieved = flops_per_launch / (ms_l / n_l / 1000.0) / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tf32_peak, "unit": "TFLOP/s",
                "frac": achieved / tf32_peak, "kernel": dom, "launches_per_step": n_l / args.steps,
                "ms_per_launch": ms_l / n_l, "algorithmic_flops_per_launch": flops_per_launch,
                "peak_kind": f"tf32 dense = {peaks_src} bf16 burst x 1.1/2.25 (nominal ratio); each fp32 "
                             "product is three tf32 products (split operands), not credited",
                "traffic": ncu_traffic(dom)}
    return {"metric": "SATA prefill backward tokens/s (dq, dk, dv)", "value": value, "unit": "tokens/s",
            "steps": args.steps, "ms_per_step": ms / args.steps,
            "workload": f"{w.name}: B={w.B} H={w.H} N={w.N} d_K={w.d_K} d_V={w.d_V} P={w.P} F={w.F}; "
                        f"dy N(0,1) fp32; the step recomputes the forward on the prefill's path",
            "l2": "L2 flushed (256 MB write) before each timed step",
            "roofline": roof, "gpu_launches": sum(n for n, _ in stats.values()),
            "kernel_ms": {k_: {"launches": n, "ms": t} for k_, (n, t) in stats.items()}}


def bench_decode(torch, sata, wl, args, world, dev, stream, peaks, peaks_src):
    """The decode workload as stated: the seeded per-head inputs of workloads.py,
    an N-token prefill into the state, then every decode step timed.  Warm-up
    steps run first on the same state, which is then rebuilt by the prefill."""
    w = wl.WORKLOADS[args.decode_workload]
    (q, k, v), (qs, ks, vs) = wl.make_inputs(w)
    D = w.steps if args.decode_steps is None else min(args.decode_steps, w.steps)
    q, k, v = q.to(dev), k.to(dev), v.to(dev)
    qs, ks, vs = qs[:D].to(dev), ks[:D].to(dev), vs[:D].to(dev)
    st = sata.State(w.B, w.H, w.d_K, w.d_V, w.P, device=dev, stream=stream)
    outs = torch.empty((D, w.B, w.H, w.d_V), dtype=torch.float32, device=dev)

    def rebuild():
        sata.sata_state_init(st.st, w.B, w.H, w.d_K, w.d_V, w.P, st.S, st.Z, stream)
        with torch.cuda.stream(stream):
            sata.prefill(q, k, v, P=w.P, state=st, stream=stream)

    rebuild()
    for i in range(min(8, D)):
        sata.sata_decode_step(st.st, qs[i], ks[i], vs[i], outs[i])
    rebuild()
    torch.cuda.synchronize()
    it = [0]

    def step():
        i = it[0]
        it[0] += 1
        sata.sata_decode_step(st.st, qs[i], ks[i], vs[i], outs[i])

    sata.sata_reset_kernel_stats()
    sata.sata_set_option(sata.SATA_OPT_TIME_KERNELS, 1)
    ms = timed(torch, world, step, D, 0, stream)
    stats = sata.sata_kernel_stats()
    sata.sata_set_option(sata.SATA_OPT_TIME_KERNELS, 0)
    if sata.sata_sync_status(stream) != 0:
        raise RuntimeError("device status after decode")
    value = job_throughput(w.B, D, world, ms)
    F = w.F
    state_bytes = 8 * F * (w.d_V + 1) * w.B * w.H          # read + write, fp32
    io_bytes = w.B * w.H * (2 * (2 * w.d_K + w.d_V) + 4 * w.d_V)
    n_l, ms_l = stats.get("decode_stream", (0, 0.0))
    roof = None
    if n_l:
        gbs = (state_bytes + io_bytes) / (ms_l / n_l / 1000.0) / 1e9
        roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": gbs / peaks["hbm_gbs"], "kernel": "decode_stream", "ms_per_launch": ms_l / n_l,
                "algorithmic_bytes_per_launch": state_bytes + io_bytes,
                "peak_kind": f"{peaks_src} HBM copy bandwidth",
                "traffic": ncu_traffic("decode_stream")}
    return {"metric": "SATA decode tokens/s", "value": value, "unit": "tokens/s", "steps": D,
            "ms_per_step": ms / D,
            "workload": f"{w.name}: B={w.B} H={w.H} d_K={w.d_K} d_V={w.d_V} P={w.P} F={F}, state from a "
                        f"{w.N}-token prefill, then steps 1..{D} timed; seeded per-head N(0,1) bf16 inputs",
            "l2": f"state {state_bytes / 2 / 1e9:.2f} GB > 126 MB L2", "roofline": roof,
            "gpu_launches": sum(n for n, _ in stats.values()),
            "kernel_ms": {k_: {"launches": n, "ms": t} for k_, (n, t) in stats.items()}}


if __name__ == "__main__":
    sys.exit(main())

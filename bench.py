"""Benchmark of FiX attention forward + backward on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2]
                    [--impl fix|reference] [--algo auto|simt|tc]

A step is one pass of the whole hot path over one batch of synthetic input:
fix_attn_fwd (training mode: saves o, m, rstd) then fix_attn_bwd, i.e. gate
prefix sums, attention forward with the fused RMSNorm, RMSNorm backward, dq,
dk/dv/dG and the reverse cumsum of dG.  Inputs are resident in HBM before the
timed region; L2 (126 MB) is flushed by writing a 256 MB buffer before every
timed step, outside the step's CUDA events.  Each step is timed on the
launching stream; the job time is the max over ranks.

Metric: FiX attention fwd+bwd TFLOP/s (causal), counting 2*B*Hq*T^2*D for
the forward (4*B*Hq*T^2*D/2; packed sequences use sum L_i^2) and 3.5x that
for forward + backward.  The forward alone is reported beside it.

Multi-GPU: every (sequence, head) unit is independent, so each rank runs its
own copy of the workload (weak scaling, no data-path collective); only the
timings are reduced.

``--impl reference`` times the fp64 CPU oracle (test infrastructure, as it
stands) on the host cores over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FiX attn fwd & fwd+bwd TFLOP/s (causal) and % of B200 dense BF16 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def fwd_flops(seqlens, Hq, Dk, Dv):
    """Causal attention FLOPs of the forward: 2 matmuls over the causal half,
    2*Hq*sum(L^2)*D (D = (Dk + Dv) / 2 when they differ)."""
    D = (Dk + Dv) / 2.0
    return 2.0 * Hq * sum(float(L) * L for L in seqlens) * D


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sms, maxes, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        try:
            lines = open(self.path).read().strip().splitlines()
        except OSError:
            lines = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxes.append(float(parts[2]))
            except ValueError:
                continue
            for name, val in zip(names, parts[5:9]):
                if val.lower() in ("active", "1"):
                    reasons.add(name)
        if self.path:
            os.unlink(self.path)
        if not sms:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxes),
                "reasons": sorted(reasons), "samples": len(sms)}


# ------------------------------------------------------------------ CPU oracle

class OracleSampler:
    """Times the fp64 oracle (forward + analytic backward, as it stands) on
    (sequence, q-head) units of a workload with a process pool on the host
    cores.  A sample is ``units`` units (default: one per worker)."""

    def __init__(self, case):
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        from oracle import fix_ref
        self.fix_ref = fix_ref
        for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
            os.environ[var] = "1"
        q, k, v, g, w, dy = (fix_ref.to64(case[x]) for x in ("q", "k", "v", "g", "w", "dy"))
        grp = case["Hq"] // case["Hkv"]
        segs = ([(b, 0, case["T"]) for b in range(case["B"])] if case["cu_seqlens"] is None
                else [(0, s0, L) for s0, L in zip(
                    [sum(case["seqlens"][:i]) for i in range(len(case["seqlens"]))],
                    case["seqlens"])])
        self.jobs, self.flops = [], []
        for b, st, L in segs:
            for h in range(case["Hq"]):
                kv = h // grp
                sl = slice(st, st + L)
                self.jobs.append((q[b, sl, h], k[b, sl, kv], v[b, sl, kv], g[b, sl, kv], w,
                                  dy[b, sl, h], case["scale"], case["eps"]))
                self.flops.append(3.5 * fwd_flops([L], 1, case["Dk"], case["Dv"]))
        self.workers = max(1, len(os.sched_getaffinity(0)))
        self.pool = ProcessPoolExecutor(max_workers=self.workers,
                                        mp_context=mp.get_context("spawn"))
        list(self.pool.map(abs, range(self.workers)))        # start the workers
        self.next = 0

    def run(self, units=None):
        """Runs one sample; returns (flop/s, seconds, units, description)."""
        n = units or self.workers
        idx = [(self.next + i) % len(self.jobs) for i in range(n)]
        self.next = (self.next + n) % len(self.jobs)
        t0 = time.perf_counter()
        list(self.pool.map(self.fix_ref._bwd_job, [self.jobs[i] for i in idx]))
        dt = time.perf_counter() - t0
        fl = sum(self.flops[i] for i in idx)
        desc = (f"{n} of {len(self.jobs)} (sequence, q-head) units per sample, fp64 forward + "
                f"analytic backward, {min(self.workers, n)} processes")
        return fl / dt, dt, n, desc

    def close(self):
        self.pool.shutdown()


# ------------------------------------------------------------------ ranks

def max_over_ranks(values, device=None):
    """Element-wise maximum of this rank's timings (ms) over the process group
    (the job is as slow as its slowest rank); the values themselves when no
    group is initialised or it has one rank."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(x) for x in values]
    t = torch.tensor([float(x) for x in values], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t]


def job_tflops(world, flops_per_step, steps, max_ms):
    """Whole-job throughput under weak scaling: every rank runs `steps` steps of
    `flops_per_step`, and the job takes the slowest rank's `max_ms`."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--impl", default="fix", choices=["fix", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    args = ap.parse_args()

    import torch
    import synth

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.workload(args.workload)
    workload_name = f"workload {args.workload}: {wl.name}"

    if args.impl == "reference":
        if rank != 0:
            return 0
        case = synth.draw(wl)
        if case["dy"] is None:
            case["dy"] = torch.randn(case["B"], case["T"], case["Hq"], case["Dv"],
                                     generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
        sampler = OracleSampler(case)
        rates, desc = [], ""
        for i in range(args.warmup + args.steps):
            fps, dt, n, desc = sampler.run()
            if i >= args.warmup:
                rates.append(fps)
        sampler.close()
        val = statistics.median(rates) / 1e12
        info = (None, min(sampler.workers, len(sampler.jobs)), desc)
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": True, "dtype": "f64", "data": "synthetic",
                "config": {"workload": workload_name},
                "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": info[1],
                                 "kind": "oracle", "sample": info[2]},
                "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0},
                "vs_baseline": None}
        print(json.dumps(line))
        return 0

    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)

    from gated_softmax_attention_fp32_b200 import fixattn

    case = synth.draw(wl)
    if case["dy"] is None:      # forward-only workloads still time fwd + bwd
        case["dy"] = torch.randn(case["B"], case["T"], case["Hq"], case["Dv"],
                                 generator=torch.Generator().manual_seed(1)).to(torch.bfloat16)
    names = ("q", "k", "v", "g", "w", "dy")
    host = {n: case[n].contiguous().pin_memory() for n in names}
    dv_ = {n: host[n].to(dev, non_blocking=True) for n in names}
    cu = case["cu_seqlens"].to(dev) if case["cu_seqlens"] is not None else None
    cu_host = case["cu_seqlens"]
    torch.cuda.synchronize()
    q, k, v, g, w, dy = (dv_[n] for n in names)
    B, T, Hq, Hkv, Dk, Dv = case["B"], case["T"], case["Hq"], case["Hkv"], case["Dk"], case["Dv"]
    eps = case["eps"]

    p, _ = fixattn.make_problem(q, k, v, cu, cu_host, None, eps, torch.bfloat16, args.algo)
    ws = torch.empty(fixattn.fix_attn_workspace_bytes(p, True), device=dev, dtype=torch.uint8)
    y = torch.empty(B, T, Hq, Dv, device=dev, dtype=torch.bfloat16)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(g),
             torch.empty_like(w))
    nst = len(fixattn.STAGES)
    flush = torch.empty(256 * 1024 * 1024, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream()

    def step(events=None):
        yy, saved = fixattn.fix_attn_fwd(q, k, v, g, w, cu, cu_host, None, eps, save=True,
                                         algo=args.algo, workspace=ws, out=y, events=events)
        fixattn.fix_attn_bwd(q, k, v, g, w, dy, saved, cu, cu_host, None, eps, algo=args.algo,
                             workspace=ws, events=events, out=grads, reuse_forward_workspace=True)
        return saved

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nst)] for _ in range(args.steps)]
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    for e in [x for row in ev for x in row]:     # torch creates the CUDA event lazily
        e.record(stream)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
    smi_id = vis.split(",")[local].strip() if vis else str(local)
    # eager steps with the per-stage events (stage times, forward time)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)                     # evict L2 outside the timed step
        starts[i].record(stream)
        step(ev[i])
        ends[i].record(stream)
    torch.cuda.synchronize()
    eager_ms = sum(s.elapsed_time(e) for s, e in zip(starts, ends)) / args.steps
    stage_ms = {name: statistics.mean(ev[i][2 * j].elapsed_time(ev[i][2 * j + 1])
                                      for i in range(args.steps))
                for j, name in enumerate(fixattn.STAGES)}
    # the step as one CUDA graph (the library's calls are stream-ordered and
    # capturable): its replays are the timed region, free of host launch gaps
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph, launch = torch.cuda.CUDAGraph(), "one CUDA graph per step (fix_attn_fwd + fix_attn_bwd)"
    try:
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
    except Exception as exc:                      # capture refused: time the eager calls
        graph, launch = None, f"eager calls (graph capture failed: {type(exc).__name__})"
        torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(smi_id) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)                 # evict L2 outside the timed step
            starts[i].record(stream)
            if graph is not None:
                graph.replay()
            else:
                step()
            ends[i].record(stream)
        torch.cuda.synchronize()
    clk = clocks.summary()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    tot_ms = sum(step_ms)
    fwd_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][3]) for i in range(args.steps))
    tot_ms, fwd_ms = max_over_ranks([tot_ms, fwd_ms], dev)
    ms_per_step = tot_ms / args.steps

    f_fwd = fwd_flops(case["seqlens"], Hq, Dk, Dv)
    f_step = 3.5 * f_fwd
    value = job_tflops(world, f_step, args.steps, tot_ms)
    fwd_tflops = job_tflops(world, f_fwd, 1, fwd_ms)

    # ---- end to end through host buffers (pinned), same metric
    e2e_ms = []
    out_host = {"dq": torch.empty(q.shape, dtype=q.dtype, pin_memory=True),
                "dk": torch.empty(k.shape, dtype=k.dtype, pin_memory=True),
                "dv": torch.empty(v.shape, dtype=v.dtype, pin_memory=True),
                "dg": torch.empty(g.shape, dtype=g.dtype, pin_memory=True),
                "dw": torch.empty(w.shape, dtype=w.dtype, pin_memory=True),
                "y": torch.empty(y.shape, dtype=y.dtype, pin_memory=True)}
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())
    for i in range(args.e2e_steps + 1):
        s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.fill_(i & 0xFF)
        s_ev.record(stream)
        for n in names:
            dv_[n].copy_(host[n], non_blocking=True)
        step()
        for key, dst in zip(("dq", "dk", "dv", "dg", "dw"), grads):
            out_host[key].copy_(dst, non_blocking=True)
        out_host["y"].copy_(y, non_blocking=True)
        e_ev.record(stream)
        torch.cuda.synchronize()
        if i > 0:
            e2e_ms.append(s_ev.elapsed_time(e_ev))
    e2e_tot, = max_over_ranks([sum(e2e_ms)], dev)
    e2e_val = job_tflops(world, f_step, len(e2e_ms), e2e_tot)

    # ---- roofline of the dominant kernel stage
    pk, pk_kind = peaks()
    attn = {k_: stage_ms[k_] for k_ in ("fwd_attn", "bwd_dq", "bwd_dkv")}
    dom = max(attn, key=attn.get)
    # algorithmic FLOPs per launch of the dominant kernel (2*Hq*sumL^2*D per
    # pair of causal GEMMs): forward QK^T and PV (1x); dk/dv kernel S, dP,
    # dV, dK (2x); dq kernel dQ only (0.5x: its S and dP are recomputation)
    share = {"fwd_attn": 1.0, "bwd_dq": 0.5, "bwd_dkv": 2.0}[dom]
    achieved = share * f_fwd / (stage_ms[dom] * 1e-3) / 1e12
    peak = pk.get("bf16_tflops_sustained" if args.steps * ms_per_step > 2000 else "bf16_tflops")
    ncu_traffic = None
    prof = os.path.join(ROOT, "profiles", "roofline_traffic.txt")
    if os.path.exists(prof):
        try:
            tr = dict(line.split(None, 1) for line in open(prof)
                      if line.strip() and not line.startswith("#"))
            tr = {key: val.strip() for key, val in tr.items()}
            if tr.get("kernel_stage") == dom and tr.get("workload") == str(args.workload) and \
                    tr.get("algo") == args.algo:
                ncu_traffic = int(tr["bytes_per_launch"])
        except (OSError, ValueError, KeyError):
            pass
    # a bounded device wait that expired would leave its status in the workspace
    dev_status = fixattn.fix_attn_device_status(ws)
    p_bwd, _k = fixattn.make_problem(q, k, v, cu, cu_host, None, eps, torch.bfloat16, args.algo)
    p_bwd.flags = fixattn.FIX_FLAG_REUSE_FWD_WORKSPACE     # as the timed backward runs
    gpu_launches = args.steps * (fixattn.fix_attn_kernel_count(p, False) +
                                 fixattn.fix_attn_kernel_count(p_bwd, True))

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_name, "B": B, "T": T, "Hq": Hq, "Hkv": Hkv,
                   "Dk": Dk, "Dv": Dv, "algo": args.algo,
                   "l2": "flushed (256 MB write) before every timed step",
                   "flops_per_step": f_step, "parallelism": f"{world} independent replicas",
                   "launch": launch},
        "eager_ms_per_step": eager_ms,
        "fwd_tflops": fwd_tflops,
        "fwd_frac_of_peak": fwd_tflops / pk["bf16_tflops"],
        "frac_of_peak": value / pk["bf16_tflops"] / world,
        "stage_ms": stage_ms,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": ncu_traffic,
                     "peak_source": pk_kind},
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": gpu_launches,
        "clocks": clk,
        "device_status": fixattn.status_string(dev_status),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sampler = OracleSampler(case)
        rates, secs, desc = [], 0.0, ""
        while secs < 12.0 and len(rates) < 8:
            fps, dt, n, desc = sampler.run()
            rates.append(fps)
            secs += dt
        sampler.close()
        line["cpu_baseline"] = {"value": statistics.median(rates) / 1e12, "unit": "TFLOP/s",
                                "cores": min(sampler.workers, len(sampler.jobs)),
                                "kind": "oracle",
                                "sample": desc + f"; median of {len(rates)} samples"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0 if dev_status == 0 else 3


if __name__ == "__main__":
    sys.exit(main())

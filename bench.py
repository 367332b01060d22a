"""Benchmark of FiX attention forward + backward on one B200 per rank.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 2]
                    [--impl fix|reference] [--algo auto|simt|tc]

A step is one pass of the whole hot path over one batch of synthetic input.
For the training workloads (2, 3, 5, 6) that is fix_attn_fwd (training mode:
saves o, m, rstd) then fix_attn_bwd, i.e. gate prefix sums, attention forward
with the fused RMSNorm, RMSNorm backward, dq, dk/dv/dG and the reverse cumsum
of dG; for the forward-only workloads (1, 4) it is one inference fix_attn_fwd
and the metric is the forward's TFLOP/s.  Inputs are resident in HBM before the
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

def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown CPU"


def _oracle_rows_job(args):
    """Oracle forward of selected rows of one (sequence, q head) unit (used
    where a whole unit would take minutes: rows are independent, so this is
    the same arithmetic on fewer rows)."""
    from oracle import fix_ref
    Q, K, V, g, w, scale, eps, rows = args
    L = Q.shape[0]
    return fix_ref.forward_rows(Q[None, :, None], K[None, :, None], V[None, :, None],
                                g[None, :, None], w, 0, L, 0, rows, scale, eps)


class OracleSampler:
    """Times the fp64 oracle (forward + analytic backward, or the forward, as
    it stands) on (sequence, q-head) units of a workload with a process pool
    on the host cores.  A sample is one unit per worker.  Forward units longer
    than ``max_rows_full`` tokens run 48 rows spread over the sequence (the
    rows of the forward are independent); their FLOPs are counted per row."""

    def __init__(self, case, backward=True, max_rows_full=8192):
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        from oracle import fix_ref
        self.fix_ref = fix_ref
        for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
            os.environ[var] = "1"
        q, k, v, g, w = (fix_ref.to64(case[x]) for x in ("q", "k", "v", "g", "w"))
        dy = fix_ref.to64(case["dy"]) if backward else None
        grp = case["Hq"] // case["Hkv"]
        segs = ([(b, 0, case["T"]) for b in range(case["B"])] if case["cu_seqlens"] is None
                else [(0, s0, L) for s0, L in zip(
                    [sum(case["seqlens"][:i]) for i in range(len(case["seqlens"]))],
                    case["seqlens"])])
        D = (case["Dk"] + case["Dv"]) / 2.0
        self.jobs, self.flops, self.kinds = [], [], []
        for b, st, L in segs:
            for h in range(case["Hq"]):
                kv = h // grp
                sl = slice(st, st + L)
                if backward:
                    self.jobs.append((q[b, sl, h], k[b, sl, kv], v[b, sl, kv], g[b, sl, kv], w,
                                      dy[b, sl, h], case["scale"], case["eps"]))
                    self.flops.append(3.5 * fwd_flops([L], 1, case["Dk"], case["Dv"]))
                    self.kinds.append("bwd")
                elif L > max_rows_full:
                    rows = sorted({int(x) for x in
                                   [L - 1] + [int(i * (L - 1) / 47) for i in range(48)]})
                    self.jobs.append((q[b, sl, h], k[b, sl, kv], v[b, sl, kv], g[b, sl, kv], w,
                                      case["scale"], case["eps"], rows))
                    self.flops.append(sum(4.0 * (t + 1) * D for t in rows))
                    self.kinds.append("rows")
                else:
                    self.jobs.append((q[b, sl, h], k[b, sl, kv], v[b, sl, kv], g[b, sl, kv], w,
                                      case["scale"], case["eps"]))
                    self.flops.append(fwd_flops([L], 1, case["Dk"], case["Dv"]))
                    self.kinds.append("fwd")
        self.backward = backward
        self.workers = max(1, len(os.sched_getaffinity(0)))
        self.cores = min(self.workers, len(self.jobs))
        self.pool = ProcessPoolExecutor(max_workers=self.workers,
                                        mp_context=mp.get_context("spawn"))
        list(self.pool.map(abs, range(self.workers)))        # start the workers
        self.next = 0

    def run(self, units=None):
        """Runs one sample; returns (flop/s, seconds, units, description)."""
        n = units or self.workers
        idx = [(self.next + i) % len(self.jobs) for i in range(n)]
        self.next = (self.next + n) % len(self.jobs)
        fns = {"bwd": self.fix_ref._bwd_job, "fwd": self.fix_ref._fwd_job,
               "rows": _oracle_rows_job}
        t0 = time.perf_counter()
        futs = [self.pool.submit(fns[self.kinds[i]], self.jobs[i]) for i in idx]
        for f in futs:
            f.result()
        dt = time.perf_counter() - t0
        fl = sum(self.flops[i] for i in idx)
        kinds = sorted({self.kinds[i] for i in idx})
        what = {"bwd": "fp64 forward + analytic backward of whole units",
                "fwd": "fp64 forward of whole units",
                "rows": "fp64 forward of 48 rows per unit"}
        desc = (f"{n} unit evaluations per sample over the workload's {len(self.jobs)} "
                f"(sequence, q-head) units, {'; '.join(what[k_] for k_ in kinds)}, "
                f"{min(self.workers, n)} processes on {cpu_model()}")
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


# ------------------------------------------------------------------ bytes

def stage_bytes(case, training):
    """Bytes each HBM-bound stage must move by its own contract (every input
    read once, every output written once; chunk-level tables of a few KB and
    the dk/dv partial-sum round trip are left out), per call.

      fwd_prefix  g (4) + v (2) read, L (4) and the three 16-bit value
                  operands (6) written: 16 B per (token, kv head, channel)
      bwd_pre     pass 1 reads o (4), dy (2), writes do (4); pass 2 reads do
                  (4), writes the three 16-bit dO operands (6): 20 B per
                  (token, q head, channel); v (2) read, A (4) written, L (4)
                  read: 10 B per kv element; q, k rows for P_tt (2 B per
                  element); m, rstd read, P_tt written (12 B per row)
      bwd_finish  L, A (8) + v (2) read, dG (4) + dv (2) written per kv
                  element, dk (2) per kv key element, do (4) per q element,
                  P_tt (4) per row
      bwd_dg      dG read by the totals and the scan (8), dg written (4):
                  12 B per kv element
    """
    N = case["B"] * case["T"]
    Hq, Hkv, Dk, Dv = case["Hq"], case["Hkv"], case["Dk"], case["Dv"]
    nq, nk = N * Hq * Dv, N * Hkv * Dv
    out = {"fwd_prefix": 16 * nk}
    if training:
        out["bwd_pre"] = 20 * nq + 10 * nk + 2 * N * (Hq + Hkv) * Dk + 12 * N * Hq
        out["bwd_finish"] = 16 * nk + 2 * N * Hkv * Dk + 4 * nq + 4 * N * Hq
        out["bwd_dg"] = 12 * nk
    return out


# ------------------------------------------------------------------ main

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", type=int, default=2)
    ap.add_argument("--impl", default="fix", choices=["fix", "reference"])
    ap.add_argument("--algo", default="auto", choices=["auto", "simt", "tc"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--clock-window-s", type=float, default=1.0,
                    help="seconds of untimed replays, inside the clock sampling window, "
                         "right before the timed steps")
    args = ap.parse_args()

    import torch
    import synth

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    wl = synth.workload(args.workload)
    training = wl.backward
    workload_name = f"workload {args.workload}: {wl.name}"

    if args.impl == "reference":
        if rank != 0:
            return 0
        case = synth.draw(wl)
        sampler = OracleSampler(case, backward=training)
        rates, desc = [], ""
        for i in range(args.warmup + args.steps):
            fps, dt, n, desc = sampler.run()
            if i >= args.warmup:
                rates.append(fps)
        sampler.close()
        val = statistics.median(rates) / 1e12
        line = {"impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOP/s",
                "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
                "higher_is_better": True, "dtype": "f64", "data": "synthetic",
                "config": {"workload": workload_name},
                "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": sampler.cores,
                                 "kind": "oracle", "sample": desc},
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
    names = ("q", "k", "v", "g", "w") + (("dy",) if training else ())
    host = {n: case[n].contiguous().pin_memory() for n in names}
    dv_ = {n: host[n].to(dev, non_blocking=True) for n in names}
    cu = case["cu_seqlens"].to(dev) if case["cu_seqlens"] is not None else None
    cu_host = case["cu_seqlens"]
    torch.cuda.synchronize()
    q, k, v, g, w = (dv_[n] for n in ("q", "k", "v", "g", "w"))
    dy = dv_.get("dy")
    B, T, Hq, Hkv, Dk, Dv = case["B"], case["T"], case["Hq"], case["Hkv"], case["Dk"], case["Dv"]
    eps = case["eps"]

    p, _ = fixattn.make_problem(q, k, v, cu, cu_host, None, eps, torch.bfloat16, args.algo)
    ws = torch.empty(max(1, fixattn.fix_attn_workspace_bytes(p, training)), device=dev,
                     dtype=torch.uint8)
    y = torch.empty(B, T, Hq, Dv, device=dev, dtype=torch.bfloat16)
    grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(g),
             torch.empty_like(w)) if training else None
    nst = len(fixattn.STAGES)
    flush = torch.empty(256 * 1024 * 1024, device=dev, dtype=torch.uint8)
    stream = torch.cuda.current_stream()

    def step(events=None):
        if not training:
            fixattn.fix_attn_fwd(q, k, v, g, w, cu, cu_host, None, eps, save=False,
                                 algo=args.algo, workspace=ws, out=y, events=events)
            return
        yy, saved = fixattn.fix_attn_fwd(q, k, v, g, w, cu, cu_host, None, eps, save=True,
                                         algo=args.algo, workspace=ws, out=y, events=events)
        fixattn.fix_attn_bwd(q, k, v, g, w, dy, saved, cu, cu_host, None, eps, algo=args.algo,
                             workspace=ws, events=events, out=grads, reuse_forward_workspace=True)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    nstage = min(args.steps, 50)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * nst)] for _ in range(nstage)]
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
    for i in range(nstage):
        flush.fill_(i & 0xFF)                     # evict L2 outside the timed step
        step(ev[i])
    torch.cuda.synchronize()
    stage_ms = {name: statistics.mean(ev[i][2 * j].elapsed_time(ev[i][2 * j + 1])
                                      for i in range(nstage))
                for j, name in enumerate(fixattn.STAGES)}
    if not training:
        stage_ms = {k_: v_ for k_, v_ in stage_ms.items() if k_.startswith("fwd")}
    fwd_eager_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][3]) for i in range(nstage))
    # the step as one CUDA graph (the library's calls are stream-ordered and
    # capturable): its replays are the timed region, free of host launch gaps
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        step()
    stream.wait_stream(side)
    torch.cuda.synchronize()
    graph, launch = torch.cuda.CUDAGraph(), "one CUDA graph per step"
    try:
        with torch.cuda.graph(graph):
            step()
        torch.cuda.synchronize()
    except Exception as exc:                      # capture refused: time the eager calls
        graph, launch = None, f"eager calls (graph capture failed: {type(exc).__name__})"
        torch.cuda.synchronize()

    def run_once():
        if graph is not None:
            graph.replay()
        else:
            step()

    # eager (direct-call) time per step, beside the graph-replay time
    for i in range(min(args.steps, 20)):
        flush.fill_(i & 0xFF)
        starts[i].record(stream)
        step()
        ends[i].record(stream)
    torch.cuda.synchronize()
    eager_ms = statistics.mean(starts[i].elapsed_time(ends[i]) for i in range(min(args.steps, 20)))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(smi_id) as clocks:
        # untimed replays inside the sampling window: the clocks under this
        # load are the ones the timed steps run at
        t_end = time.perf_counter() + args.clock_window_s
        while time.perf_counter() < t_end:
            for _ in range(20):
                flush.fill_(1)
                run_once()
            torch.cuda.synchronize()
        for i in range(args.steps):
            flush.fill_(i & 0xFF)                 # evict L2 outside the timed step
            starts[i].record(stream)
            run_once()
            ends[i].record(stream)
        torch.cuda.synchronize()
    clk = clocks.summary()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    tot_ms = sum(step_ms)
    # forward alone as a graph (training forward for the training workloads)
    fwd_graph_ms = None
    if training:
        gf = torch.cuda.CUDAGraph()
        try:
            with torch.cuda.graph(gf):
                fixattn.fix_attn_fwd(q, k, v, g, w, cu, cu_host, None, eps, save=True,
                                     algo=args.algo, workspace=ws, out=y)
            torch.cuda.synchronize()
            fs = []
            for i in range(min(args.steps, 50)):
                flush.fill_(i & 0xFF)
                starts[i].record(stream)
                gf.replay()
                ends[i].record(stream)
            torch.cuda.synchronize()
            fwd_graph_ms = statistics.mean(starts[i].elapsed_time(ends[i])
                                           for i in range(min(args.steps, 50)))
        except Exception:
            torch.cuda.synchronize()
    else:
        fwd_graph_ms = tot_ms / args.steps
    tot_ms, fwd_ms = max_over_ranks([tot_ms, fwd_graph_ms or fwd_eager_ms], dev)
    ms_per_step = tot_ms / args.steps

    f_fwd = fwd_flops(case["seqlens"], Hq, Dk, Dv)
    f_step = 3.5 * f_fwd if training else f_fwd
    value = job_tflops(world, f_step, args.steps, tot_ms)
    fwd_tflops = job_tflops(world, f_fwd, 1, fwd_ms)

    # ---- end to end through host buffers (pinned), same metric
    e2e_ms = []
    out_host = {"y": torch.empty(y.shape, dtype=y.dtype, pin_memory=True)}
    if training:
        for key, t_ in zip(("dq", "dk", "dv", "dg", "dw"), grads):
            out_host[key] = torch.empty(t_.shape, dtype=t_.dtype, pin_memory=True)
    h2d = sum(host[n].numel() * host[n].element_size() for n in names)
    d2h = sum(t.numel() * t.element_size() for t in out_host.values())
    for i in range(args.e2e_steps + 1):
        s_ev, e_ev = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        flush.fill_(i & 0xFF)
        s_ev.record(stream)
        for n in names:
            dv_[n].copy_(host[n], non_blocking=True)
        step()
        if training:
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
    cand = ("fwd_attn", "bwd_dq", "bwd_dkv") if training else ("fwd_attn",)
    attn = {k_: stage_ms[k_] for k_ in cand}
    dom = max(attn, key=attn.get)
    # algorithmic FLOPs per launch of the dominant kernel (2*Hq*sumL^2*D per
    # pair of causal GEMMs): forward QK^T and PV (1x); dk/dv kernel S, dP,
    # dV, dK (2x); dq kernel dQ only (0.5x: its S and dP are recomputation)
    share = {"fwd_attn": 1.0, "bwd_dq": 0.5, "bwd_dkv": 2.0}[dom]
    achieved = share * f_fwd / (stage_ms[dom] * 1e-3) / 1e12
    # the kernel is timed inside a step of well under a second: burst peak
    peak = pk.get("bf16_tflops")
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
    hbm = pk.get("hbm_gbs")
    stage_gbs = {}
    for name, nbytes in stage_bytes(case, training).items():
        ms = stage_ms.get(name)
        if ms and ms > 0:
            gbs = nbytes / (ms * 1e-3) / 1e9
            stage_gbs[name] = {"bytes": nbytes, "gbs": gbs, "frac_of_hbm": gbs / hbm}
    # a bounded device wait that expired would leave its status in the workspace
    dev_status = fixattn.fix_attn_device_status(ws)
    p_bwd, _k = fixattn.make_problem(q, k, v, cu, cu_host, None, eps, torch.bfloat16, args.algo)
    p_bwd.flags = fixattn.FIX_FLAG_REUSE_FWD_WORKSPACE     # as the timed backward runs
    per_step = fixattn.fix_attn_kernel_count(p, False)
    if training:
        per_step += fixattn.fix_attn_kernel_count(p_bwd, True)
    gpu_launches = args.steps * per_step

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": workload_name, "B": B, "T": T, "Hq": Hq, "Hkv": Hkv,
                   "Dk": Dk, "Dv": Dv, "algo": args.algo,
                   "step": "fwd (training) + bwd" if training else "fwd (inference)",
                   "l2": "flushed (256 MB write) before every timed step",
                   "flops_per_step": f_step, "parallelism": f"{world} independent replicas",
                   "launch": launch},
        "eager_ms_per_step": eager_ms,
        "fwd_tflops": fwd_tflops,
        "fwd_ms": fwd_ms,
        "fwd_frac_of_peak": fwd_tflops / pk["bf16_tflops"],
        "frac_of_peak": value / pk["bf16_tflops"] / world,
        "stage_ms": stage_ms,
        "stage_gbs": stage_gbs,
        "roofline": {"bound": "tensor", "kernel": dom, "achieved": achieved, "peak": peak,
                     "unit": "TFLOP/s", "frac": achieved / peak, "traffic": ncu_traffic,
                     "peak_source": pk_kind + " (burst)"},
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": gpu_launches,
        "clocks": clk,
        "device_status": fixattn.status_string(dev_status),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sampler = OracleSampler(case, backward=training)
        rates, secs, desc = [], 0.0, ""
        while secs < 12.0 and len(rates) < 8:
            fps, dt, n, desc = sampler.run()
            rates.append(fps)
            secs += dt
        sampler.close()
        line["cpu_baseline"] = {"value": statistics.median(rates) / 1e12, "unit": "TFLOP/s",
                                "cores": sampler.cores, "kind": "oracle",
                                "sample": desc + f"; median of {len(rates)} samples"}
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0 if dev_status == 0 else 3


if __name__ == "__main__":
    sys.exit(main())

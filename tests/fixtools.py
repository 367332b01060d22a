"""Helpers for the GPU parity tests: run the CUDA path, sample the oracle."""
from __future__ import annotations

import os

import numpy as np
import torch

from oracle import fix_ref

# Parity bars (rel-L2 = ||x - ref|| / ||ref|| over a tensor).  Forward on the
# float32 output y after the RMSNorm; gradients per tensor.
FWD_REL_L2 = 5e-3
FWD_MAX_ABS = 2e-2
GRAD_REL_L2 = 1e-2


def workers():
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def rel_l2(x, ref):
    x = np.asarray(x, np.float64).ravel()
    ref = np.asarray(ref, np.float64).ravel()
    return float(np.linalg.norm(x - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs(x, ref):
    return float(np.max(np.abs(np.asarray(x, np.float64) - np.asarray(ref, np.float64))))


def to_cuda(case):
    out = {}
    for key in ("q", "k", "v", "g", "w", "dy", "cu_seqlens"):
        t = case.get(key)
        out[key] = None if t is None else t.cuda().contiguous()
    return out


def run_gpu(case, algo="auto", backward=False, y_dtype=torch.float32, reuse=True, o_gate=None,
            o_norm=True):
    """Forward (and backward) through the C ABI; returns numpy float64 dicts.
    ``reuse``: the backward reuses the forward's workspace (its gate prefix).
    ``o_gate``: a CPU bf16 tensor [B,T,Hq,Dv]; a gate g of shape [B,T,Hkv]
    runs the scalar-gate mode."""
    from gated_softmax_attention_fp32_b200 import fixattn
    t = to_cuda(case)
    z = o_gate.cuda().contiguous() if o_gate is not None else None
    cu_host = case["cu_seqlens"]
    scalar = t["g"].dim() == 3
    # one workspace for both calls, so that the device status word (where a
    # bounded device wait that expired reports) can be checked after each
    p, _keep = fixattn.make_problem(t["q"], t["k"], t["v"], t["cu_seqlens"], cu_host, None,
                                    case["eps"], y_dtype, algo, None, o_norm, scalar)
    ws = torch.empty(max(fixattn.fix_attn_workspace_bytes(p, backward), 1), device="cuda",
                     dtype=torch.uint8)
    w = t["w"] if o_norm else None
    y, saved = fixattn.fix_attn_fwd(t["q"], t["k"], t["v"], t["g"], w, t["cu_seqlens"],
                                    cu_host, None, case["eps"], y_dtype=y_dtype, save=True,
                                    algo=algo, workspace=ws, o_gate=z, o_norm=o_norm)
    assert fixattn.fix_attn_device_status(ws) == 0, "forward: device status not OK"
    res = dict(y=y, o=saved[0], m=saved[1], rstd=saved[2])
    if backward:
        dq, dk, dv, dg, dw, dz = fixattn.fix_attn_bwd(
            t["q"], t["k"], t["v"], t["g"], w, t["dy"], saved, t["cu_seqlens"], cu_host, None,
            case["eps"], algo=algo, workspace=ws, reuse_forward_workspace=reuse, o_gate=z,
            o_norm=o_norm)
        assert fixattn.fix_attn_device_status(ws) == 0, "backward: device status not OK"
        res.update(dq=dq, dk=dk, dv=dv, dg=dg)
        if dw is not None:
            res["dw"] = dw
        if dz is not None:
            res["d_o_gate"] = dz
    torch.cuda.synchronize()
    return {k: v.float().cpu().numpy().astype(np.float64) for k, v in res.items()}


def oracle_full(case, backward=False, o_gate=None, o_norm=True):
    args = (case["q"], case["k"], case["v"], case["g"], case["w"])
    seqlens = case["seqlens"] if case["cu_seqlens"] is not None else None
    f = fix_ref.forward(*args, seqlens, None, case["eps"], workers(), norm=o_norm, o_gate=o_gate)
    if backward:
        f.update(fix_ref.backward(*args, case["dy"], seqlens, None, case["eps"], workers(),
                                  norm=o_norm, o_gate=o_gate))
    return f


def segments(case):
    """(batch index, start token, length) of every sequence."""
    if case["cu_seqlens"] is None:
        return [(b, 0, case["T"]) for b in range(case["B"])]
    out, s0 = [], 0
    for L in case["seqlens"]:
        out.append((0, s0, L))
        s0 += L
    return out


def sample_rows(L, n, rng):
    """Rows of a length-L sequence: first, last 8, tile edges and random."""
    if L == 0:
        return []
    rows = {0, L - 1}
    rows.update(range(max(0, L - 8), L))
    for e in (127, 128, 129, 255, 256):
        if e < L:
            rows.add(e)
    rows.update(int(x) for x in rng.integers(0, L, size=n))
    return sorted(rows)


def sequence_case(case, b, s0, L):
    """The inputs of one sequence of ``case`` as a dense B = 1 problem (the
    operator never mixes sequences, so its outputs on these rows are the same
    as in the packed problem)."""
    out = dict(case)
    for key in ("q", "k", "v", "g", "dy"):
        if case.get(key) is not None:
            out[key] = case[key][b:b + 1, s0:s0 + L].contiguous()
    out.update(B=1, T=L, cu_seqlens=None, seqlens=[L])
    return out


def _suffix_job(args):
    q, k, v, g, w, dy, L, R, eps = args
    return fix_ref.suffix_backward(q, k, v, g, w, dy, 0, L, 0, R, None, eps)


def oracle_suffix(case, picks, R):
    """dk, dv, dg of the last R key rows of (b, start, L, kv) picks, from the
    oracle's suffix backward, one pick per process of a spawn pool.  Each job
    gets only its sequence and its kv group (so kv = 0 inside the job)."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    grp = case["Hq"] // case["Hkv"]
    jobs = []
    for b, s0, L, kv in picks:
        sl = slice(s0, s0 + L)
        hs = slice(kv * grp, (kv + 1) * grp)
        jobs.append((case["q"][b:b + 1, sl, hs], case["k"][b:b + 1, sl, kv:kv + 1],
                     case["v"][b:b + 1, sl, kv:kv + 1], case["g"][b:b + 1, sl, kv:kv + 1],
                     case["w"], case["dy"][b:b + 1, sl, hs], L, min(R, L), case["eps"]))
    n = max(1, min(workers(), len(jobs)))
    if n == 1:
        return [_suffix_job(j) for j in jobs]
    with ProcessPoolExecutor(max_workers=n, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(_suffix_job, jobs))

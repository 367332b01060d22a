"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Small and odd shapes (several 128-token chunks, ragged tails, every head dim,
GQA, Dk != Dv, packed sequences with empty and length-1 members, fast-decay
channels, the README's positive randn gate) are compared element by element
with the full oracle; the five workloads at full size are compared on
sampled rows, which the oracle computes exactly one by one.

Bars: forward rel-L2 <= 5e-3 and max-abs <= 2e-2 on float32 y; gradients
dq, dk, dv, dg, dw rel-L2 <= 1e-2 per tensor.
"""
import numpy as np
import pytest
import torch

import synth
from fixtools import (FWD_MAX_ABS, FWD_REL_L2, GRAD_REL_L2, max_abs, oracle_full,
                      oracle_suffix, rel_l2, run_gpu, sample_rows, segments, sequence_case,
                      workers)
from oracle import fix_ref

pytestmark = pytest.mark.gpu

GRADS = ("dq", "dk", "dv", "dg", "dw")


def check_fwd(y, ref, tag=""):
    e, m = rel_l2(y, ref), max_abs(y, ref)
    assert e <= FWD_REL_L2 and m <= FWD_MAX_ABS, f"{tag} y rel-L2 {e:.2e} max-abs {m:.2e}"


def check_grad(name, x, ref, tag=""):
    """rel-L2 <= 1e-2, measured against max(||ref||, 1e-4 * sqrt(numel)).

    The floor (1e-4 RMS per element, far below the O(0.01..1) size of these
    gradients) only matters where a gradient vanishes analytically up to
    eps-sized terms: e.g. dq of a sequence's first row, whose only key has
    weight exactly 1, so dq there is proportional to the RMSNorm eps and both
    sides hold rounding noise of the cancelling terms."""
    x = np.asarray(x, np.float64); ref = np.asarray(ref, np.float64)
    den = max(np.linalg.norm(ref.ravel()), 1e-4 * np.sqrt(ref.size))
    e = np.linalg.norm((x - ref).ravel()) / den
    assert e <= GRAD_REL_L2, f"{tag} {name} rel-L2 {e:.2e}"


SMALL = {
    "T1": dict(B=1, T=1, Hq=1, Hkv=1, Dk=64, Dv=64),
    # fewer than 128 tokens in all: the exact CUDA-core kernels
    "B2-T63-gqa-exact": dict(B=2, T=63, Hq=4, Hkv=2, Dk=64, Dv=64),
    # one ragged chunk per sequence on the tensor-core kernels
    "B3-T63-gqa": dict(B=3, T=63, Hq=4, Hkv=2, Dk=64, Dv=64),
    "B2-T100-D128": dict(B=2, T=100, Hq=2, Hkv=1, Dk=128, Dv=128),
    "T129-D32": dict(B=1, T=129, Hq=2, Hkv=2, Dk=32, Dv=32),
    "B2-T300-D16": dict(B=2, T=300, Hq=4, Hkv=1, Dk=16, Dv=16),
    "T257-Dk64-Dv128": dict(B=1, T=257, Hq=2, Hkv=1, Dk=64, Dv=128),
    "T200-Dk128-Dv64": dict(B=1, T=200, Hq=3, Hkv=3, Dk=128, Dv=64),
    "T520-D128": dict(B=1, T=520, Hq=2, Hkv=1, Dk=128, Dv=128),
    "varlen": dict(B=1, T=0, Hq=4, Hkv=2, Dk=64, Dv=64, seqlens=[0, 1, 130, 7, 255, 0, 64, 300]),
    "fast-channels": dict(B=1, T=300, Hq=2, Hkv=1, Dk=64, Dv=64, g_mean=1.0, channel_bias_std=2.5),
    "T520-D128-gqa-fast-channels": dict(B=1, T=520, Hq=4, Hkv=2, Dk=128, Dv=128, g_mean=1.0,
                                        channel_bias_std=2.5),
    "readme-randn-gate": dict(B=1, T=200, Hq=2, Hkv=1, Dk=64, Dv=64, raw_gate=True, g_mean=0.0),
}


def out_of_range_channels(case):
    """(chunk, kv head, channel) triples whose in-chunk gate range exceeds
    the decay split's float range (half-range above 80): the kernels handle
    their diagonal terms exactly in fp32."""
    g = case["g"].double().numpy()
    n = 0
    for b, T in enumerate(case["seqlens"] if case["cu_seqlens"] is None else [None]):
        seqs = ([(b, 0, T)] if T is not None else
                [(0, int(a), int(e)) for a, e in zip(case["cu_seqlens"][:-1], case["cu_seqlens"][1:])])
        for bb, a, e in seqs:
            for c0 in range(a, e, 128):
                L = np.cumsum(g[bb, c0:min(c0 + 128, e)], axis=0)
                rng = L.max(axis=0) - L.min(axis=0)
                n += int((rng / 2 > 80).sum())
    return n


@pytest.mark.parametrize("name", ["T520-D128", "fast-channels", "varlen"])
def test_backward_reusing_forward_workspace_is_identical(cuda_lib, name):
    """FIX_FLAG_REUSE_FWD_WORKSPACE: the backward reads the forward's gate
    prefix results instead of recomputing them (for "fast-channels" that
    includes the out-of-range channel flags); the gradients are bit-identical
    to a backward that recomputes."""
    case = synth.make_case(**SMALL[name], seed=7)
    a = run_gpu(case, "auto", backward=True, reuse=True)
    b = run_gpu(case, "auto", backward=True, reuse=False)
    for key in ("y",) + tuple(GRADS):
        assert np.array_equal(a[key], b[key]), (name, key)


@pytest.mark.parametrize("algo", ["auto", "simt"])
@pytest.mark.parametrize("name", list(SMALL))
def test_small_shapes(cuda_lib, name, algo):
    case = synth.make_case(**SMALL[name], seed=42)
    if "fast-channels" in name:
        assert out_of_range_channels(case) > 0, "the case must exercise the exact diagonal terms"
    gpu = run_gpu(case, algo, backward=True)
    ref = oracle_full(case, backward=True)
    check_fwd(gpu["y"], ref["y"], name)
    for key in GRADS:
        check_grad(key, gpu[key], ref[key], name)
    # the saved tensors are consistent with y
    w = case["w"].double().numpy()
    assert rel_l2(gpu["o"] * gpu["rstd"][..., None] * w, gpu["y"]) < 1e-5


def test_bf16_output_matches_f32_output(cuda_lib):
    case = synth.make_case(1, 300, 4, 2, 64, 64, seed=1)
    a = run_gpu(case, y_dtype=torch.float32)["y"]
    b = run_gpu(case, y_dtype=torch.bfloat16)["y"]
    assert max_abs(a, b) <= np.abs(a).max() * 2 ** -8


def test_outputs_fully_written_nan_poison(cuda_lib, monkeypatch):
    """Every output and workspace byte starts as NaN / 0xFF (as FLA's test
    suite poisons torch.empty); the results must still match the oracle."""
    real_empty, real_like = torch.empty, torch.empty_like

    def poison(t):
        if t.dtype == torch.uint8:
            return t.fill_(255)
        return t.fill_(float("nan")) if t.is_floating_point() else t

    monkeypatch.setattr(torch, "empty", lambda *a, **k: poison(real_empty(*a, **k)))
    monkeypatch.setattr(torch, "empty_like", lambda *a, **k: poison(real_like(*a, **k)))
    case = synth.make_case(1, 0, 4, 2, 64, 64, seqlens=[0, 3, 200, 1, 129], seed=3)
    gpu = run_gpu(case, backward=True)
    monkeypatch.undo()
    ref = oracle_full(case, backward=True)
    for key, val in gpu.items():
        assert np.isfinite(val).all(), key
    check_fwd(gpu["y"], ref["y"])
    for key in GRADS:
        check_grad(key, gpu[key], ref[key])


def test_device_status_ok_after_calls(cuda_lib):
    from gated_softmax_attention_fp32_b200 import fixattn
    case = synth.make_case(1, 256, 2, 1, 64, 64, seed=4)
    t = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case.items()}
    p, _ = fixattn.make_problem(t["q"], t["k"], t["v"])
    ws = torch.empty(fixattn.fix_attn_workspace_bytes(p, True), device="cuda", dtype=torch.uint8)
    y, saved = fixattn.fix_attn_fwd(t["q"], t["k"], t["v"], t["g"], t["w"], workspace=ws)
    assert fixattn.fix_attn_device_status(ws) == 0
    fixattn.fix_attn_bwd(t["q"], t["k"], t["v"], t["g"], t["w"], t["dy"], saved, workspace=ws)
    assert fixattn.fix_attn_device_status(ws) == 0


# --------------------------------------------------------------- workloads

def test_workload1_forward_full(cuda_lib):
    case = synth.draw(synth.workload(1))
    gpu = run_gpu(case)
    ref = oracle_full(case)
    check_fwd(gpu["y"], ref["y"], "workload 1")


def test_workload2_forward_backward_full(cuda_lib):
    case = synth.draw(synth.workload(2))
    gpu = run_gpu(case, backward=True)
    ref = oracle_full(case, backward=True)
    check_fwd(gpu["y"], ref["y"], "workload 2")
    for key in GRADS:
        check_grad(key, gpu[key], ref[key], "workload 2")


def _sampled_forward(case, gpu, rows_per_seq, heads, seed=0):
    rng = np.random.default_rng(seed)
    ys, refs = [], []
    for b, s0, L in segments(case):
        for h in heads:
            rows = sample_rows(L, rows_per_seq, rng)
            if not rows:
                continue
            r = fix_ref.forward_rows(case["q"], case["k"], case["v"], case["g"], case["w"],
                                     (b, s0), L, h, rows, None, case["eps"])
            refs.append(r["y"])
            ys.append(gpu["y"][b, [s0 + t for t in rows], h])
    return np.concatenate(ys), np.concatenate(refs)


def _sampled_dq(case, gpu, rows_per_seq, heads, seed=1):
    rng = np.random.default_rng(seed)
    xs, refs = [], []
    for b, s0, L in segments(case):
        for h in heads:
            rows = sample_rows(L, rows_per_seq, rng)
            if not rows:
                continue
            refs.append(fix_ref.dq_rows(case["q"], case["k"], case["v"], case["g"], case["w"],
                                        case["dy"], s0, L, h, rows, None, case["eps"], b=b))
            xs.append(gpu["dq"][b, [s0 + t for t in rows], h])
    return np.concatenate(xs), np.concatenate(refs)


def _suffix(case, gpu, picks, R):
    res = oracle_suffix(case, picks, R)
    out = {k: ([], []) for k in ("dk", "dv", "dg")}
    for (b, s0, L, kv), r in zip(picks, res):
        sl = slice(s0 + L - min(R, L), s0 + L)
        for key in out:
            out[key][0].append(gpu[key][b, sl, kv])
            out[key][1].append(r[key])
    return {k: (np.concatenate(a), np.concatenate(b)) for k, (a, b) in out.items()}


def _properties(case, gpu):
    for key, val in gpu.items():
        assert np.isfinite(val).all(), key
    if "dg" in gpu:
        scale = np.sqrt((gpu["dg"] ** 2).mean())
        for b, s0, L in segments(case):
            if L:
                assert np.abs(gpu["dg"][b, s0]).max() <= 1e-3 * max(scale, 1e-12) * np.sqrt(L)


def test_workload3_varlen_sampled(cuda_lib):
    """Packed sequences of 2817, 6892, 6576 and 99 tokens.  The two short ones
    get the full oracle (every output and gradient of their rows); the two
    long ones sampled forward / dq rows and the last 384 key rows of dk, dv,
    dg for the first and last kv head: those keys span three 128-token
    chunks, so their later-block dk/dv parts and the combine of several
    partial slots are compared, not only the diagonal.  dw is a sum over all
    rows: it is checked against sum(dy * y / w), which holds exactly for the
    float32 y whose rows are compared with the oracle above."""
    case = synth.draw(synth.workload(3))
    gpu = run_gpu(case, backward=True)
    _properties(case, gpu)
    segs = segments(case)
    short = [s for s in segs if s[2] <= 3000]
    long_ = [s for s in segs if s[2] > 3000]
    assert short and long_
    for b, s0, L in short:
        sub = sequence_case(case, b, s0, L)
        ref = oracle_full(sub, backward=True)
        sl = slice(s0, s0 + L)
        check_fwd(gpu["y"][b, sl], ref["y"][0], f"workload 3 seq len {L}")
        for key in ("dq", "dk", "dv", "dg"):
            check_grad(key, gpu[key][b, sl], ref[key][0], f"workload 3 seq len {L}")
    y, ref = _sampled_forward(case, gpu, 24, range(case["Hq"]))
    check_fwd(y, ref, "workload 3")
    x, ref = _sampled_dq(case, gpu, 6, range(0, case["Hq"], 3))
    check_grad("dq", x, ref, "workload 3")
    picks = [(b, s0, L, kv) for (b, s0, L) in long_ for kv in (0, case["Hkv"] - 1)]
    for key, (x, ref) in _suffix(case, gpu, picks, 384).items():
        check_grad(key, x, ref, "workload 3 (last 384 keys)")
    w = case["w"].double().numpy()
    dy = case["dy"].double().numpy()
    dw_from_y = (dy * gpu["y"] / w).sum(axis=(0, 1, 2))
    check_grad("dw", gpu["dw"], dw_from_y, "workload 3 (sum dy*y/w)")


def test_workload4_long_context_sampled(cuda_lib):
    case = synth.draw(synth.workload(4))
    gpu = run_gpu(case)
    _properties(case, gpu)
    y, ref = _sampled_forward(case, gpu, 8, range(case["Hq"]))
    check_fwd(y, ref, "workload 4")


def test_workload5_full(cuda_lib):
    # 128 (sequence, head) units of T = 4096: the full oracle takes about a
    # minute on 16 host cores, so every gradient is compared element-wise
    case = synth.draw(synth.workload(5))
    gpu = run_gpu(case, backward=True)
    _properties(case, gpu)
    ref = oracle_full(case, backward=True)
    check_fwd(gpu["y"], ref["y"], "workload 5")
    for key in GRADS:
        check_grad(key, gpu[key], ref[key], "workload 5")


# ------------------------------------------ o_gate, o_norm = False, scalar gate
# FiX README "Quick Start" (o_norm, o_norm_weight, o_gate arguments) and the
# Forgetting Transformer abstract (scalar forget gates); readings in the
# oracle's header.

OPTION_SHAPES = {
    "T300-D64-gqa": dict(B=1, T=300, Hq=4, Hkv=2, Dk=64, Dv=64),
    "B2-T257-D128": dict(B=2, T=257, Hq=2, Hkv=1, Dk=128, Dv=128),
    "varlen-D64": dict(B=1, T=0, Hq=2, Hkv=1, Dk=64, Dv=64, seqlens=[0, 1, 130, 7, 255]),
    "T129-D32": dict(B=1, T=129, Hq=2, Hkv=2, Dk=32, Dv=32),
}


def _gate(case, seed):
    gen = torch.Generator().manual_seed(seed)
    return torch.randn(case["B"], case["T"], case["Hq"], case["Dv"], generator=gen).to(
        torch.bfloat16)


def _check_all(gpu, ref, tag, o_norm=True):
    check_fwd(gpu["y"], ref["y"], tag)
    keys = ["dq", "dk", "dv", "dg"] + (["dw"] if o_norm else []) + \
        (["d_o_gate"] if "d_o_gate" in ref else [])
    for key in keys:
        check_grad(key, gpu[key], ref[key], tag)


@pytest.mark.parametrize("algo", ["auto", "simt"])
@pytest.mark.parametrize("name", list(OPTION_SHAPES))
def test_output_gate(cuda_lib, name, algo):
    case = synth.make_case(**OPTION_SHAPES[name], seed=51)
    z = _gate(case, 52)
    gpu = run_gpu(case, algo, backward=True, o_gate=z)
    ref = oracle_full(case, backward=True, o_gate=z)
    _check_all(gpu, ref, f"{name} o_gate")


@pytest.mark.parametrize("algo", ["auto", "simt"])
@pytest.mark.parametrize("name", list(OPTION_SHAPES))
def test_no_norm(cuda_lib, name, algo):
    case = synth.make_case(**OPTION_SHAPES[name], seed=53)
    gpu = run_gpu(case, algo, backward=True, o_norm=False)
    ref = oracle_full(case, backward=True, o_norm=False)
    _check_all(gpu, ref, f"{name} no norm", o_norm=False)


@pytest.mark.parametrize("algo", ["auto", "simt"])
@pytest.mark.parametrize("name", list(OPTION_SHAPES))
def test_scalar_gate(cuda_lib, name, algo):
    case = synth.make_case(**OPTION_SHAPES[name], seed=54)
    case = dict(case, g=case["g"][..., 0].contiguous())     # one gate per (token, kv head)
    gpu = run_gpu(case, algo, backward=True)
    ref = oracle_full(case, backward=True)
    assert gpu["dg"].shape == ref["dg"].shape == tuple(case["g"].shape)
    _check_all(gpu, ref, f"{name} scalar gate")


def test_all_options_together_workload2_shape(cuda_lib):
    """Scalar gate, no norm and an output gate on the README's example shape
    (B2 T2048 H8/4 D128), every output and gradient against the full oracle."""
    case = synth.draw(synth.workload(2))
    case = dict(case, g=case["g"][..., 0].contiguous())
    z = _gate(case, 55)
    gpu = run_gpu(case, backward=True, o_gate=z, o_norm=False)
    ref = oracle_full(case, backward=True, o_gate=z, o_norm=False)
    _check_all(gpu, ref, "workload 2 shape, all options", o_norm=False)


# ------------------------------------------------------------------ decode
# One new query per sequence against its (k, v, g) cache: y must equal row
# L - 1 of the forward of the same sequence.  Cache slots past each length
# hold NaN, so any read beyond L would show.

def _decode_case(lengths, Tmax, Hq, Hkv, D, seed, scalar=False):
    B = len(lengths)
    case = synth.make_case(B, Tmax, Hq, Hkv, D, D, seed=seed)
    if scalar:
        case = dict(case, g=case["g"][..., 0].contiguous())
    return case


def _decode_ref(case, lengths, o_gate=None, o_norm=True):
    ys = []
    for b, L in enumerate(lengths):
        sub = sequence_case(case, b, 0, L)
        z = None if o_gate is None else o_gate[b:b + 1, None].expand(1, L, -1, -1).contiguous()
        ref = oracle_full(sub, o_gate=z, o_norm=o_norm)
        ys.append(ref["y"][0, L - 1])
    return np.stack(ys)


@pytest.mark.parametrize("opts", [dict(), dict(gate=True), dict(o_norm=False),
                                  dict(scalar=True, gate=True)])
def test_decode_matches_last_forward_row(cuda_lib, opts):
    from gated_softmax_attention_fp32_b200 import fixattn
    lengths, Tmax = [1, 70, 300, 129], 320
    case = _decode_case(lengths, Tmax, 4, 2, 64, 61, opts.get("scalar", False))
    B = len(lengths)
    qd = torch.stack([case["q"][b, L - 1] for b, L in enumerate(lengths)])
    kc, vc, gc = (case[x].clone() for x in ("k", "v", "g"))
    for b, L in enumerate(lengths):
        kc[b, L:] = float("nan"); vc[b, L:] = float("nan"); gc[b, L:] = float("nan")
    z = None
    if opts.get("gate"):
        z = torch.randn(B, 4, 64, generator=torch.Generator().manual_seed(62)).to(torch.bfloat16)
    o_norm = opts.get("o_norm", True)
    y = fixattn.fix_attn_decode(qd.cuda(), kc.cuda(), vc.cuda(), gc.cuda(),
                                torch.tensor(lengths, dtype=torch.int32).cuda(),
                                case["w"].cuda() if o_norm else None, eps=case["eps"],
                                y_dtype=torch.float32, o_norm=o_norm,
                                o_gate=None if z is None else z.cuda())
    torch.cuda.synchronize()
    ref = _decode_ref(case, lengths, z, o_norm)
    check_fwd(y.double().cpu().numpy(), ref, f"decode {opts}")


def test_decode_long_context_rows(cuda_lib):
    """Workload 4's shape (T = 32768, H 32/8, D 128) as a decode of its last
    token, and of a shorter cache, against the oracle's rows."""
    from gated_softmax_attention_fp32_b200 import fixattn
    case = synth.draw(synth.workload(4))
    T = case["T"]
    lengths = [T, 20000]
    kc = case["k"].expand(2, -1, -1, -1).contiguous()
    vc = case["v"].expand(2, -1, -1, -1).contiguous()
    gc = case["g"].expand(2, -1, -1, -1).contiguous()
    qd = torch.stack([case["q"][0, L - 1] for L in lengths])
    y = fixattn.fix_attn_decode(qd.cuda(), kc.cuda(), vc.cuda(), gc.cuda(),
                                torch.tensor(lengths, dtype=torch.int32).cuda(),
                                case["w"].cuda(), eps=case["eps"], y_dtype=torch.float32)
    torch.cuda.synchronize()
    for b, L in enumerate(lengths):
        for h in (0, 13, 31):
            r = fix_ref.forward_rows(case["q"], case["k"], case["v"], case["g"], case["w"],
                                     (0, 0), L, h, [L - 1], None, case["eps"])
            check_fwd(y[b, h].double().cpu().numpy()[None], r["y"], f"decode L={L} h={h}")


# ------------------------------------------------------------------ autograd
def test_autograd_wrapper_matches_direct_calls(cuda_lib):
    """fix_attn (the README's call, as a torch.autograd.Function) gives the
    same y and gradients as the direct forward/backward calls, bit for bit,
    with the device status checked after each."""
    from gated_softmax_attention_fp32_b200 import fixattn
    case = synth.make_case(1, 300, 4, 2, 64, 64, seed=21)
    t = {k: case[k].cuda() for k in ("q", "k", "v", "g", "w", "dy")}
    leaves = {k: t[k].clone().requires_grad_(True) for k in ("q", "k", "v", "g", "w")}
    y = fixattn.fix_attn(leaves["q"], leaves["k"], leaves["v"], leaves["g"], leaves["w"])
    y.backward(t["dy"])
    yd, saved = fixattn.fix_attn_fwd(t["q"], t["k"], t["v"], t["g"], t["w"], save=True)
    dq, dk, dv, dg, dw, _ = fixattn.fix_attn_bwd(t["q"], t["k"], t["v"], t["g"], t["w"], t["dy"],
                                                 saved)
    torch.cuda.synchronize()
    assert torch.equal(y.detach(), yd)
    for name, ref in (("q", dq), ("k", dk), ("v", dv), ("g", dg), ("w", dw)):
        assert torch.equal(leaves[name].grad, ref), name

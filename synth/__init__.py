"""Seeded synthetic inputs for FiX attention workloads.

This module only draws random tensors: it holds none of the operator's
arithmetic, so both the fp64 oracle (``oracle/``) and the CUDA path may be fed
from it.  Every tensor is created on the CPU with a ``torch.Generator`` seeded
explicitly, in one fixed draw order:

    [varlen lengths] -> q -> k -> v -> x -> g = logsigmoid(x) -> w -> dy

q, k, v and dy are standard normal rounded to bf16; the gate logit x is fp32
normal with the workload's mean and standard deviation and g = logsigmoid(x)
(so g <= 0, a forget gate in log space).  The output-norm weight w is either
ones or bf16 N(1, 0.1).

Shapes follow the FiX README ("Quick Start"): q [B,T,Hq,Dk], k [B,T,Hkv,Dk],
v and g [B,T,Hkv,Dv]; packed sequences use B = 1 plus int64 ``cu_seqlens``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch
import torch.nn.functional as F

__all__ = ["Case", "WORKLOADS", "workload", "make_case", "draw"]


@dataclasses.dataclass(frozen=True)
class Case:
    """Shape and distribution of one synthetic FiX problem."""

    B: int
    T: int
    Hq: int
    Hkv: int
    Dk: int
    Dv: int
    g_mean: float
    g_std: float
    w_kind: str = "ones"            # "ones" | "normal" (bf16 N(1, 0.1))
    backward: bool = True
    seqlens: Optional[tuple] = None  # packed sequence lengths (B must be 1)
    varlen_draw: Optional[tuple] = None  # (total, lo, hi): lengths drawn U{lo..hi}
    channel_bias_std: float = 0.0   # per-channel shift of x (heterogeneous decay)
    raw_gate: bool = False          # g = x itself (the README example draws g = randn)
    eps: float = 1e-6
    seed: int = 0
    name: str = ""


# The workloads of the FiX operator studied here.  Sizes are those of the
# FiX README's Quick Start example (B2, T2048, 8 q heads over 4 kv heads, D128)
# and of typical long-context / training shapes.
WORKLOADS = {
    1: Case(1, 256, 2, 1, 64, 64, 3.0, 1.0, "ones", backward=False,
            name="fwd B1 T256 Hq2 Hkv1 D64"),
    2: Case(2, 2048, 8, 4, 128, 128, 3.0, 1.0, "normal", backward=True,
            name="fwd+bwd B2 T2048 Hq8 Hkv4 D128"),
    3: Case(1, 16384, 16, 4, 128, 128, 4.0, 1.5, "ones", backward=True,
            varlen_draw=(16384, 128, 8192),
            name="varlen fwd+bwd N16384 Hq16 Hkv4 D128"),
    4: Case(1, 32768, 32, 8, 128, 128, 5.0, 1.0, "ones", backward=False,
            name="fwd B1 T32768 Hq32 Hkv8 D128"),
    5: Case(8, 4096, 16, 16, 64, 64, 2.0, 2.0, "normal", backward=True,
            name="fwd+bwd B8 T4096 Hq16 Hkv16 D64"),
    # workload 2's shape with heterogeneous decay: a per-channel shift of the
    # gate logit (std 2.5) makes about a fifth of the channels forget fast
    # enough that their in-chunk range exceeds the decay split's float range
    6: Case(2, 2048, 8, 4, 128, 128, 1.0, 1.0, "normal", backward=True,
            channel_bias_std=2.5,
            name="fwd+bwd B2 T2048 Hq8 Hkv4 D128, fast-decay channels (bias std 2.5)"),
}


def workload(n: int) -> Case:
    return WORKLOADS[n]


def _draw_lengths(gen: torch.Generator, total: int, lo: int, hi: int) -> list:
    lens = []
    acc = 0
    while acc < total:
        n = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
        lens.append(n)
        acc += n
    lens[-1] -= acc - total          # truncate the last one to fit
    return lens


def draw(case: Case) -> dict:
    """Draw all tensors of ``case`` on the CPU (seeded, fixed order).

    Returns a dict with q, k, v (bf16), g (fp32), w (bf16), dy (bf16 or None),
    cu_seqlens (int64 or None), seqlens (list of int) and scalar metadata.
    """
    gen = torch.Generator().manual_seed(case.seed)
    seqlens = None
    if case.varlen_draw is not None:
        total, lo, hi = case.varlen_draw
        seqlens = _draw_lengths(gen, total, lo, hi)
    elif case.seqlens is not None:
        seqlens = list(case.seqlens)
    if seqlens is not None:
        assert case.B == 1, "packed sequences use B = 1"
        T = int(sum(seqlens))
    else:
        T = case.T
    B = case.B
    q = torch.randn(B, T, case.Hq, case.Dk, generator=gen).to(torch.bfloat16)
    k = torch.randn(B, T, case.Hkv, case.Dk, generator=gen).to(torch.bfloat16)
    v = torch.randn(B, T, case.Hkv, case.Dv, generator=gen).to(torch.bfloat16)
    x = torch.randn(B, T, case.Hkv, case.Dv, generator=gen) * case.g_std + case.g_mean
    if case.channel_bias_std:
        bias = torch.randn(case.Hkv, case.Dv, generator=gen) * case.channel_bias_std
        x = x + bias
    g = (x if case.raw_gate else F.logsigmoid(x)).to(torch.float32).contiguous()
    if case.w_kind == "ones":
        w = torch.ones(case.Dv, dtype=torch.bfloat16)
    else:
        w = (torch.randn(case.Dv, generator=gen) * 0.1 + 1.0).to(torch.bfloat16)
    dy = None
    if case.backward:
        dy = torch.randn(B, T, case.Hq, case.Dv, generator=gen).to(torch.bfloat16)
    cu = None
    if seqlens is not None:
        cu = torch.zeros(len(seqlens) + 1, dtype=torch.int64)
        cu[1:] = torch.cumsum(torch.tensor(seqlens, dtype=torch.int64), 0)
    return dict(q=q, k=k, v=v, g=g, w=w, dy=dy, cu_seqlens=cu,
                seqlens=seqlens if seqlens is not None else [T] * B,
                B=B, T=T, Hq=case.Hq, Hkv=case.Hkv, Dk=case.Dk, Dv=case.Dv,
                eps=case.eps, scale=case.Dk ** -0.5)


def make_case(B, T, Hq, Hkv, Dk, Dv, *, g_mean=3.0, g_std=1.0, w_kind="normal",
              backward=True, seqlens=None, channel_bias_std=0.0, raw_gate=False, eps=1e-6,
              seed=0) -> dict:
    """Convenience wrapper: build a ``Case`` and draw it."""
    c = Case(B, T, Hq, Hkv, Dk, Dv, g_mean, g_std, w_kind, backward,
             tuple(seqlens) if seqlens is not None else None, None,
             channel_bias_std, raw_gate, eps, seed)
    return draw(c)

"""Brute-force FiX forward in pure Python loops (tiny inputs only).

TEST INFRASTRUCTURE ONLY (see ``oracle/fix_ref.py``).  This is the operator's
definition typed out a second time with scalar loops and ``math.exp``: for
every output element it walks s = 0..t and multiplies the decay factors
exp(g_r[c]) for r = s+1..t one by one, instead of forming prefix sums.  It
exists to pin the vectorised oracle and, through finite differences of it,
the oracle's analytic backward.
"""
from __future__ import annotations

import math

__all__ = ["brute_forward", "brute_loss"]


def brute_forward(q, k, v, g, w, seqlens, scale, eps, m_fixed=None, norm=True, z=None):
    """q[b][t][h][d] nested lists (or arrays indexable the same way).

    Returns y as nested lists [B][T][Hq][Dv] and m [B][T][Hq].
    ``m_fixed`` (same shape as m) replaces the row max when given.  ``g`` may
    be [B][T][Hkv] (one gate per token and kv head, for every channel).
    ``norm = False``: y = o / sum_s p instead of the RMSNorm; ``z``
    [B][T][Hq][Dv]: y is multiplied by z / (1 + exp(-z)).
    """
    B = len(q)
    T = len(q[0])
    Hq = len(q[0][0]) if T else 0
    Dk = len(q[0][0][0]) if T else 0
    Hkv = len(v[0][0]) if T else 0
    Dv = len(v[0][0][0]) if T else 0
    grp = Hq // Hkv if Hkv else 1
    scalar = T > 0 and not hasattr(g[0][0][0], "__len__")

    def gate(b, t, kv, c):
        return float(g[b][t][kv]) if scalar else float(g[b][t][kv][c])
    y = [[[[0.0] * Dv for _ in range(Hq)] for _ in range(T)] for _ in range(B)]
    mm = [[[0.0] * Hq for _ in range(T)] for _ in range(B)]
    if B == 1 and seqlens is not None:
        segs, s0 = [], 0
        for L in seqlens:
            segs.append((0, s0, L)); s0 += L
    else:
        segs = [(b, 0, T) for b in range(B)]
    for b, s0, L in segs:
        for h in range(Hq):
            kv = h // grp
            for ti in range(L):
                t = s0 + ti
                logits = []
                for si in range(ti + 1):
                    s = s0 + si
                    acc = 0.0
                    for d in range(Dk):
                        acc += float(q[b][t][h][d]) * float(k[b][s][kv][d])
                    logits.append(scale * acc)
                mt = max(logits) if m_fixed is None else float(m_fixed[b][t][h])
                mm[b][t][h] = mt
                o = [0.0] * Dv
                psum = 0.0
                for si in range(ti + 1):
                    s = s0 + si
                    p = math.exp(logits[si] - mt)
                    psum += p
                    for c in range(Dv):
                        dec = 1.0
                        for ri in range(si + 1, ti + 1):
                            dec *= math.exp(gate(b, s0 + ri, kv, c))
                        o[c] += p * dec * float(v[b][s][kv][c])
                ms = sum(x * x for x in o) / Dv
                r = 1.0 / math.sqrt(ms + eps)
                for c in range(Dv):
                    y[b][t][h][c] = o[c] * r * float(w[c]) if norm else o[c] / psum
                    if z is not None:
                        zz = float(z[b][t][h][c])
                        y[b][t][h][c] *= zz / (1.0 + math.exp(-zz))
    return y, mm


def brute_loss(q, k, v, g, w, dy, seqlens, scale, eps, m_fixed=None, norm=True, z=None):
    """sum(dy * y) with the brute-force forward (for finite differences)."""
    y, _ = brute_forward(q, k, v, g, w, seqlens, scale, eps, m_fixed, norm, z)
    tot = 0.0
    for b in range(len(y)):
        for t in range(len(y[b])):
            for h in range(len(y[b][t])):
                for c in range(len(y[b][t][h])):
                    tot += float(dy[b][t][h][c]) * y[b][t][h][c]
    return tot

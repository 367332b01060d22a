"""FiX attention oracle: a plain, slow, fp64 CPU implementation.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` use it.  It shares no code with the CUDA library.

What it computes (FiX: "Introducing Fine-grained Forget Gate into Softmax
Attention"; poster abstract: the softmax denominator is redundant under the
RMSNorm that follows, so the forgetting becomes an element-wise multiplication
on the value vectors; README "Quick Start": g has v's shape, GQA heads,
``o_norm`` RMSNorm with a [Dv] weight, ``cu_seqlens`` packing):

    per sequence, q head h, kv head kv(h) = h // (Hq / Hkv), 0 <= s <= t < L:
      S_ts    = scale * <q_t, k_s>
      m_t     = max_{s<=t} S_ts                   (per-row shift, a constant)
      P_ts    = exp(S_ts - m_t)
      G_t[c]  = sum_{r=0..t} g_r[c]               (restarts at each sequence)
      D_ts[c] = exp(G_t[c] - G_s[c]) = exp(sum_{r=s+1..t} g_r[c])
      o_t[c]  = sum_{s<=t} P_ts * D_ts[c] * v_s[c]
      rstd_t  = (mean_c o_t[c]^2 + eps)^(-1/2)
      y_t     = o_t * rstd_t * w

Readings of points the pages leave open (each is listed with its reason in
the repository's design notes): the decay of pair (t, s) sums g over r in
(s, t], so g at a sequence's first token never matters; m_t is the exact
causal row max of the logits and is a constant (stop-gradient) in the
backward; consecutive q heads share a kv head; scale = Dk^-1/2 by default.

The backward is the analytic one, written pair by pair (no block
factorisation, no cancellation-prone identity):

      dw     = sum_t dy_t * n_t                    n_t = o_t * rstd_t
      dn_t   = dy_t * w
      do_t   = rstd_t * (dn_t - n_t * mean_c(dn_t * n_t))
      W_ts   = P_ts * D_ts
      dv_s  += W_ts * do_t
      dP_ts  = sum_c do_t[c] D_ts[c] v_s[c]
      dS_ts  = P_ts * dP_ts
      dq_t   = scale * sum_s dS_ts k_s ;   dk_s = scale * sum_t dS_ts q_t
      dG_t  += do_t * o_t ;                dG_s -= W_ts * do_t * v_s
      dg_r   = sum_{t>=r} dG_t                    (within the sequence)
    dk, dv, dg are summed over the q heads of each kv group.

Options of the same call (FiX README, "Quick Start": ``o_norm``,
``o_norm_weight``, ``o_gate``; Forgetting Transformer abstract: scalar
forget gates), each a reading of points the pages leave open:

  o_norm = False   no RMSNorm; the output is the attention average with the
                   ordinary softmax denominator, o_t / l_t with
                   l_t = sum_{s<=t} P_ts (so g = 0 gives causal softmax
                   attention), and m_t drops out exactly
  o_gate z         y <- y * swish(z) = y * z * sigmoid(z), after the norm and
                   its weight (the output-gate form of the library FiX is
                   forked from); z has y's shape [B,T,Hq,Dv]
  scalar gate      g of shape [B,T,Hkv]: one forget gate per (token, kv head),
                   the same for every value channel; FiX with g broadcast over
                   the channels, and dg is the channel sum of that gradient

Pins (see tests/test_oracle.py): brute-force loops, finite differences,
library identities (g = 0 is RMSNorm of ordinary causal softmax attention;
channel-constant g is Forgetting-Transformer attention), closed forms and
invariants.
"""
from __future__ import annotations

import os
from typing import Optional, Sequence

import numpy as np

__all__ = [
    "unit_forward", "unit_backward", "forward", "backward",
    "forward_rows", "dq_rows", "suffix_backward", "to64", "swish", "swish_grad",
]


def to64(x) -> np.ndarray:
    """Convert a torch tensor / array to a float64 numpy array (exact for bf16, fp32)."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        import torch  # local: only for the dtype conversion
        return x.to(torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


# --------------------------------------------------------------------------
# One (sequence, q-head) unit
# --------------------------------------------------------------------------

def swish(z):
    """z * sigmoid(z)."""
    return z / (1.0 + np.exp(-z))


def swish_grad(z):
    """d/dz of z * sigmoid(z) = sigmoid(z) * (1 + z * (1 - sigmoid(z)))."""
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def unit_forward(Q, K, V, g, w, scale, eps, m_fixed=None, norm=True, z=None):
    """Forward of one (sequence, q head) unit in fp64.

    Q [L,Dk], K [L,Dk], V [L,Dv], g [L,Dv] (the kv head's tensors), w [Dv].
    ``m_fixed`` (optional [L]) replaces the row max; used by finite-difference
    tests that hold the per-row shift constant.  ``norm = False``: y is
    o_t / l_t (no RMSNorm, no weight); ``z`` [L,Dv]: y <- y * swish(z).
    Returns y, o, m, rstd, P, G.
    """
    L = Q.shape[0]
    Dv = V.shape[1]
    if L == 0:
        z = np.zeros((0, Dv))
        return z, z.copy(), np.zeros(0), np.zeros(0), np.zeros((0, 0)), z.copy()
    G = np.cumsum(g, axis=0)                       # inclusive prefix sum
    S = scale * (Q @ K.T)
    causal = np.tri(L, dtype=bool)                 # s <= t
    Sm = np.where(causal, S, -np.inf)
    m = Sm.max(axis=1) if m_fixed is None else np.asarray(m_fixed, np.float64)
    P = np.exp(Sm - m[:, None])                    # exp(-inf) = 0 above the diagonal
    o = np.empty((L, Dv))
    for t in range(L):
        D = np.exp(G[t][None, :] - G[: t + 1])     # D_ts[c], s = 0..t
        o[t] = np.einsum("s,sc,sc->c", P[t, : t + 1], D, V[: t + 1])
    rstd = 1.0 / np.sqrt((o * o).mean(axis=1) + eps)
    y = o * rstd[:, None] * w[None, :]
    if not norm:
        y = o / P.sum(axis=1)[:, None]             # softmax denominator l_t
    if z is not None:
        y = y * swish(z)
    return y, o, m, rstd, P, G


def unit_backward(Q, K, V, g, w, dy, scale, eps, norm=True, z=None):
    """Analytic backward of one (sequence, q head) unit in fp64.

    Returns dQ [L,Dk], dK [L,Dk], dV [L,Dv], dg [L,Dv], dw [Dv], dz [L,Dv]
    (None without an output gate) for this q head (dK, dV, dg are this
    head's share of the kv head's gradients).  With ``norm = False`` the
    softmax denominator is part of the function: P is normalised and
    dS_ts = P_ts (dP_ts - sum_c do_t[c] o_t[c]), the exact derivative.
    """
    L, Dk = Q.shape
    Dv = V.shape[1]
    if L == 0:
        return (np.zeros((0, Dk)), np.zeros((0, Dk)), np.zeros((0, Dv)),
                np.zeros((0, Dv)), np.zeros(Dv), None if z is None else np.zeros((0, Dv)))
    y, o, m, rstd, P, G = unit_forward(Q, K, V, g, w, scale, eps)
    if z is not None:
        dy_gated = dy
        dy = dy_gated * swish(z)                   # gradient of the ungated output
    if norm:
        n = o * rstd[:, None]
        u = n * w[None, :]                         # ungated output
        dw = (dy * n).sum(axis=0)
        dn = dy * w[None, :]
        do = rstd[:, None] * (dn - n * (dn * n).mean(axis=1, keepdims=True))
    else:
        ell = P.sum(axis=1)
        P = P / ell[:, None]                       # normalised weights
        o = o / ell[:, None]
        u = o
        dw = np.zeros(Dv)
        do = dy
    dz = None if z is None else dy_gated * u * swish_grad(z)
    dV = np.zeros((L, Dv))
    dG = np.zeros((L, Dv))
    dP = np.zeros((L, L))
    for t in range(L):
        D = np.exp(G[t][None, :] - G[: t + 1])     # [t+1, Dv]
        W = P[t, : t + 1, None] * D                # W_ts[c]
        dV[: t + 1] += W * do[t][None, :]
        dP[t, : t + 1] = (D * V[: t + 1]) @ do[t]
        dG[t] += do[t] * o[t]
        dG[: t + 1] -= W * do[t][None, :] * V[: t + 1]
    dS = P * dP
    if not norm:
        dS = P * (dP - (do * o).sum(axis=1)[:, None])
    dQ = scale * (dS @ K)
    dK = scale * (dS.T @ Q)
    dg = np.cumsum(dG[::-1], axis=0)[::-1]         # dg_r = sum_{t>=r} dG_t
    return dQ, dK, dV, dg, dw, dz


# --------------------------------------------------------------------------
# Whole problems: batches / packed sequences, GQA heads, optional process pool
# --------------------------------------------------------------------------

def _segments(B, T, seqlens):
    """Yield (b, start, length) for every sequence."""
    if seqlens is None or B > 1:
        for b in range(B):
            yield b, 0, T
        return
    start = 0
    for L in seqlens:
        yield 0, start, int(L)
        start += int(L)


def _fwd_job(args):
    Q, K, V, g, w, scale, eps = args[:7]
    norm, z = (args[7], args[8]) if len(args) > 7 else (True, None)
    y, o, m, rstd, _, _ = unit_forward(Q, K, V, g, w, scale, eps, None, norm, z)
    return y, o, m, rstd


def _bwd_job(args):
    return unit_backward(*args)


def _pool_map(fn, jobs, workers):
    if workers is None:
        workers = 1
    if workers <= 1 or len(jobs) <= 1:
        return [fn(j) for j in jobs]
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    for var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
        os.environ.setdefault(var, "1")
    with ProcessPoolExecutor(max_workers=workers, mp_context=mp.get_context("spawn")) as ex:
        return list(ex.map(fn, jobs))


def _channel_gate(g, Dv):
    """A scalar gate [B,T,Hkv] as the element-wise gate it stands for."""
    return np.repeat(g[..., None], Dv, axis=-1) if g.ndim == 3 else g


def forward(q, k, v, g, w, seqlens=None, scale=None, eps=1e-6, workers=None, norm=True,
            o_gate=None):
    """Full forward.  q [B,T,Hq,Dk], k [B,T,Hkv,Dk], v [B,T,Hkv,Dv], g
    [B,T,Hkv,Dv] (or [B,T,Hkv]: scalar gate), w [Dv], o_gate None or
    [B,T,Hq,Dv].

    ``seqlens`` (B == 1) lists packed sequence lengths.  Returns a dict of
    float64 arrays: y, o [B,T,Hq,Dv]; m, rstd [B,T,Hq].
    """
    q, k, v, g, w, o_gate = (to64(x) for x in (q, k, v, g, w, o_gate))
    B, T, Hq, Dk = q.shape
    Hkv, Dv = v.shape[2], v.shape[3]
    g = _channel_gate(g, Dv)
    assert Hq % Hkv == 0
    grp = Hq // Hkv
    if scale is None:
        scale = Dk ** -0.5
    jobs, where = [], []
    for b, s0, L in _segments(B, T, seqlens):
        for h in range(Hq):
            kv = h // grp
            sl = slice(s0, s0 + L)
            jobs.append((q[b, sl, h], k[b, sl, kv], v[b, sl, kv], g[b, sl, kv], w, scale, eps))
            if not norm or o_gate is not None:
                jobs[-1] += (norm, None if o_gate is None else o_gate[b, sl, h])
            where.append((b, sl, h))
    res = _pool_map(_fwd_job, jobs, workers)
    y = np.zeros((B, T, Hq, Dv)); o = np.zeros((B, T, Hq, Dv))
    m = np.zeros((B, T, Hq)); rstd = np.zeros((B, T, Hq))
    for (b, sl, h), (yy, oo, mm, rr) in zip(where, res):
        y[b, sl, h] = yy; o[b, sl, h] = oo; m[b, sl, h] = mm; rstd[b, sl, h] = rr
    return dict(y=y, o=o, m=m, rstd=rstd)


def backward(q, k, v, g, w, dy, seqlens=None, scale=None, eps=1e-6, workers=None, norm=True,
             o_gate=None):
    """Full analytic backward of L = sum(dy * y).  Returns dq, dk, dv, dg, dw
    (and d_o_gate with an output gate); for a scalar gate [B,T,Hkv], dg has
    that shape."""
    q, k, v, g, w, dy, o_gate = (to64(x) for x in (q, k, v, g, w, dy, o_gate))
    B, T, Hq, Dk = q.shape
    Hkv, Dv = v.shape[2], v.shape[3]
    scalar_gate = g.ndim == 3
    g = _channel_gate(g, Dv)
    grp = Hq // Hkv
    if scale is None:
        scale = Dk ** -0.5
    jobs, where = [], []
    for b, s0, L in _segments(B, T, seqlens):
        for h in range(Hq):
            kv = h // grp
            sl = slice(s0, s0 + L)
            jobs.append((q[b, sl, h], k[b, sl, kv], v[b, sl, kv], g[b, sl, kv], w,
                         dy[b, sl, h], scale, eps))
            if not norm or o_gate is not None:
                jobs[-1] += (norm, None if o_gate is None else o_gate[b, sl, h])
            where.append((b, sl, h, kv))
    res = _pool_map(_bwd_job, jobs, workers)
    dq = np.zeros_like(q); dk = np.zeros_like(k); dv = np.zeros_like(v)
    dg = np.zeros_like(g); dw = np.zeros(Dv)
    dz = None if o_gate is None else np.zeros_like(o_gate)
    for (b, sl, h, kv), (a, bk, bv, bg, bw, bz) in zip(where, res):
        dq[b, sl, h] = a
        dk[b, sl, kv] += bk
        dv[b, sl, kv] += bv
        dg[b, sl, kv] += bg
        dw += bw
        if dz is not None:
            dz[b, sl, h] = bz
    out = dict(dq=dq, dk=dk, dv=dv, dg=dg.sum(axis=-1) if scalar_gate else dg, dw=dw)
    if dz is not None:
        out["d_o_gate"] = dz
    return out


# --------------------------------------------------------------------------
# Sampled outputs for workloads too large for the full oracle.  Rows of the
# forward are independent given the inputs, so these are exact for the rows
# they return (not approximations).
# --------------------------------------------------------------------------

def _row(Qh, Kh, Vh, G, t, scale):
    s = scale * (Kh[: t + 1] @ Qh[t])
    mt = s.max()
    p = np.exp(s - mt)
    D = np.exp(G[t][None, :] - G[: t + 1])
    o = np.einsum("s,sc,sc->c", p, D, Vh[: t + 1])
    return o, mt, p, D


def forward_rows(q, k, v, g, w, start, L, h, rows, scale=None, eps=1e-6):
    """y, o, m, rstd for selected rows (0-based within the sequence) of one
    sequence [start, start+L) and q head h.  Cost O(rows * t * D)."""
    q, k, v, g, w = (to64(x) for x in (q, k, v, g, w))
    b = 0
    if q.ndim == 4 and isinstance(start, tuple):
        b, start = start
    Hq, Dk = q.shape[2], q.shape[3]
    Hkv = v.shape[2]
    kv = h // (Hq // Hkv)
    if scale is None:
        scale = Dk ** -0.5
    sl = slice(start, start + L)
    Qh, Kh, Vh = q[b, sl, h], k[b, sl, kv], v[b, sl, kv]
    G = np.cumsum(g[b, sl, kv], axis=0)
    out_y, out_o, out_m, out_r = [], [], [], []
    for t in rows:
        o, mt, _, _ = _row(Qh, Kh, Vh, G, int(t), scale)
        r = 1.0 / np.sqrt((o * o).mean() + eps)
        out_y.append(o * r * w); out_o.append(o); out_m.append(mt); out_r.append(r)
    return dict(y=np.array(out_y), o=np.array(out_o), m=np.array(out_m), rstd=np.array(out_r))


def dq_rows(q, k, v, g, w, dy, start, L, h, rows, scale=None, eps=1e-6, b=0):
    """dq for selected rows of one (sequence, q head).  Cost O(rows * t * D)."""
    q, k, v, g, w, dy = (to64(x) for x in (q, k, v, g, w, dy))
    Hq, Dk = q.shape[2], q.shape[3]
    Hkv = v.shape[2]
    kv = h // (Hq // Hkv)
    if scale is None:
        scale = Dk ** -0.5
    sl = slice(start, start + L)
    Qh, Kh, Vh = q[b, sl, h], k[b, sl, kv], v[b, sl, kv]
    G = np.cumsum(g[b, sl, kv], axis=0)
    out = []
    for t in rows:
        t = int(t)
        o, mt, p, D = _row(Qh, Kh, Vh, G, t, scale)
        r = 1.0 / np.sqrt((o * o).mean() + eps)
        n = o * r
        dn = dy[b, start + t, h] * w
        do = r * (dn - n * (dn * n).mean())
        dP = (D * Vh[: t + 1]) @ do
        out.append(scale * ((p * dP) @ Kh[: t + 1]))
    return np.array(out)


def suffix_backward(q, k, v, g, w, dy, start, L, kv, R, scale=None, eps=1e-6, b=0):
    """dk, dv, dg (summed over the kv group's q heads) for the last R rows
    of one sequence.  Needs every row t >= L-R of the forward: O(R * L * D)
    per head.  Returns arrays of shape [R, D]."""
    q, k, v, g, w, dy = (to64(x) for x in (q, k, v, g, w, dy))
    Hq, Dk = q.shape[2], q.shape[3]
    Hkv, Dv = v.shape[2], v.shape[3]
    grp = Hq // Hkv
    if scale is None:
        scale = Dk ** -0.5
    sl = slice(start, start + L)
    Kh, Vh = k[b, sl, kv], v[b, sl, kv]
    G = np.cumsum(g[b, sl, kv], axis=0)
    r0 = L - R
    dK = np.zeros((R, Dk)); dV = np.zeros((R, Dv)); dG = np.zeros((R, Dv))
    for h in range(kv * grp, (kv + 1) * grp):
        Qh = q[b, sl, h]
        for t in range(r0, L):
            o, mt, p, D = _row(Qh, Kh, Vh, G, t, scale)
            rr = 1.0 / np.sqrt((o * o).mean() + eps)
            n = o * rr
            dn = dy[b, start + t, h] * w
            do = rr * (dn - n * (dn * n).mean())
            ps, Ds = p[r0:], D[r0:]                 # key rows s in [r0, t]
            W = ps[:, None] * Ds
            dV[: t + 1 - r0] += W * do[None, :]
            dP = (Ds * Vh[r0: t + 1]) @ do
            dK[: t + 1 - r0] += scale * (ps * dP)[:, None] * Qh[t][None, :]
            dG[t - r0] += do * o
            dG[: t + 1 - r0] -= W * do[None, :] * Vh[r0: t + 1]
    dg = np.cumsum(dG[::-1], axis=0)[::-1]
    return dict(dk=dK, dv=dV, dg=dg)

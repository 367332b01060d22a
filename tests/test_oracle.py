"""Pins for the fp64 oracle, checked against things other than itself.

Each test ties the oracle to a fact the FiX pages or plain mathematics fix:
brute-force loops, finite differences, library routines (torch's scaled-dot-
product attention) for the special cases that reduce to ordinary causal
softmax attention (g = 0) and to Forgetting-Transformer attention (channel-
constant g), closed forms, and invariants of the definition.  A plausible slip
in the oracle (a dropped term, a wrong sign or index, a transposed operand)
fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import brute_forward, brute_loss, fix_ref

HERE = os.path.dirname(os.path.abspath(__file__))


def rnd(rng, *shape):
    return rng.standard_normal(shape)


def make(rng, B, T, Hq, Hkv, Dk, Dv, g_scale=1.0, g_kind="logsig"):
    q = rnd(rng, B, T, Hq, Dk)
    k = rnd(rng, B, T, Hkv, Dk)
    v = rnd(rng, B, T, Hkv, Dv)
    x = rnd(rng, B, T, Hkv, Dv) * g_scale + 1.0
    g = -np.log1p(np.exp(-x)) if g_kind == "logsig" else x
    w = 1.0 + 0.1 * rnd(rng, Dv)
    dy = rnd(rng, B, T, Hq, Dv)
    return q, k, v, g, w, dy


def relerr(a, b):
    a = np.asarray(a, np.float64); b = np.asarray(b, np.float64)
    den = np.linalg.norm(b.ravel())
    return np.linalg.norm((a - b).ravel()) / max(den, 1e-300)


# ---------------------------------------------------------------- brute force

TINY = [
    # B, T, Hq, Hkv, Dk, Dv, seqlens
    (1, 1, 1, 1, 2, 2, None),
    (1, 2, 1, 1, 4, 2, None),
    (2, 3, 2, 1, 2, 4, None),
    (1, 5, 4, 2, 4, 4, None),
    (1, 8, 2, 2, 2, 4, None),
    (1, 8, 4, 2, 2, 2, [0, 3, 0, 1, 4]),
]


@pytest.mark.parametrize("B,T,Hq,Hkv,Dk,Dv,seqlens", TINY)
def test_oracle_forward_matches_brute_force(B, T, Hq, Hkv, Dk, Dv, seqlens):
    rng = np.random.default_rng(42)
    q, k, v, g, w, _ = make(rng, B, T, Hq, Hkv, Dk, Dv)
    scale, eps = 0.7, 1e-6
    ref = fix_ref.forward(q, k, v, g, w, seqlens, scale, eps)
    yb, mb = brute_forward(q, k, v, g, w, seqlens, scale, eps)
    assert relerr(ref["y"], yb) < 1e-12
    assert np.allclose(ref["m"], np.array(mb), rtol=0, atol=1e-12)


def test_oracle_forward_matches_brute_force_positive_gate():
    # the README's example draws g = randn, i.e. some g > 0
    rng = np.random.default_rng(7)
    q, k, v, g, w, _ = make(rng, 1, 6, 2, 1, 3, 3, g_kind="raw")
    ref = fix_ref.forward(q, k, v, g, w, None, 0.5, 1e-6)
    yb, _ = brute_forward(q, k, v, g, w, None, 0.5, 1e-6)
    assert relerr(ref["y"], yb) < 1e-12


# ------------------------------------------------------- finite differences

def _fd_check(B, T, Hq, Hkv, Dk, Dv, seqlens, eps, hold_m, seed):
    rng = np.random.default_rng(seed)
    q, k, v, g, w, dy = make(rng, B, T, Hq, Hkv, Dk, Dv)
    scale = 0.8
    grads = fix_ref.backward(q, k, v, g, w, dy, seqlens, scale, eps)
    m0 = fix_ref.forward(q, k, v, g, w, seqlens, scale, eps)["m"] if hold_m else None
    args = dict(q=q, k=k, v=v, g=g, w=w)
    h = 1e-5
    for name, gname in [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("w", "dw")]:
        x = args[name]
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            old = x[idx]
            x[idx] = old + h
            lp = brute_loss(args["q"], args["k"], args["v"], args["g"], args["w"], dy,
                            seqlens, scale, eps, m0)
            x[idx] = old - h
            lm = brute_loss(args["q"], args["k"], args["v"], args["g"], args["w"], dy,
                            seqlens, scale, eps, m0)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        err = relerr(grads[gname], fd)
        assert err < 1e-7, (gname, err)


@pytest.mark.parametrize("case", [
    (1, 4, 2, 1, 3, 3, None),
    (1, 7, 2, 2, 2, 3, [3, 0, 4]),
    (2, 3, 4, 2, 2, 2, None),
])
def test_backward_matches_finite_differences_m_held(case):
    # m_t held at its base value: the backward treats the row shift as a constant
    _fd_check(*case, eps=1e-2, hold_m=True, seed=3)


def test_backward_matches_finite_differences_eps0_m_free():
    # at eps = 0 the output does not depend on the row shift at all, so the
    # stop-gradient backward must equal the true derivative with m free
    _fd_check(1, 5, 2, 1, 3, 3, None, eps=0.0, hold_m=False, seed=5)


# ----------------------------------------------------------- library identities

def _sdpa(q, k, v, mask=None, scale=1.0):
    """torch SDPA on fp64 CPU tensors; q [T,H,D] layout per batch."""
    Q = torch.from_numpy(q).permute(1, 0, 2)[None]
    K = torch.from_numpy(k).permute(1, 0, 2)[None]
    V = torch.from_numpy(v).permute(1, 0, 2)[None]
    if mask is None:
        out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=scale)
    else:
        out = torch.nn.functional.scaled_dot_product_attention(
            Q, K, V, attn_mask=torch.from_numpy(mask)[None], scale=scale)
    return out[0].permute(1, 0, 2).numpy()


def _rms(o, w, eps):
    return o / np.sqrt((o * o).mean(-1, keepdims=True) + eps) * w


def test_zero_gate_is_rmsnorm_of_causal_softmax_attention():
    rng = np.random.default_rng(11)
    T, Hq, Hkv, D = 37, 4, 2, 8
    q, k, v, _, w, _ = make(rng, 1, T, Hq, Hkv, D, D)
    g = np.zeros((1, T, Hkv, D))
    scale = D ** -0.5
    kr = np.repeat(k[0], Hq // Hkv, axis=1)
    vr = np.repeat(v[0], Hq // Hkv, axis=1)
    sd = _sdpa(q[0], kr, vr, scale=scale)                      # normalised attention
    # eps = 0: FiX equals RMSNorm(softmax attention) * w exactly
    y0 = fix_ref.forward(q, k, v, g, w, None, scale, 0.0)["y"][0]
    assert relerr(y0, _rms(sd, w, 0.0)) < 1e-12
    # eps > 0: o carries the softmax denominator l_t = sum_s exp(S_ts - m_t)
    out = fix_ref.forward(q, k, v, g, w, None, scale, 1e-6)
    S = scale * np.einsum("thd,shd->hts", q[0], kr)
    Sm = np.where(np.tri(T, dtype=bool)[None], S, -np.inf)
    ell = np.exp(Sm - Sm.max(-1, keepdims=True)).sum(-1).T    # [T, H]
    assert relerr(out["o"][0], sd * ell[..., None]) < 1e-12
    assert relerr(out["y"][0], _rms(sd * ell[..., None], w, 1e-6)) < 1e-12


def _fox_mask(a):
    """Forgetting-Transformer additive bias: sum of the log forget gates
    strictly after the key up to the query (the FoX abstract: forget gates
    down-weight the unnormalised scores); -inf above the diagonal."""
    T = a.shape[0]
    M = np.full((T, T), -np.inf)
    for t in range(T):
        for s in range(t + 1):
            M[t, s] = sum(a[r] for r in range(s + 1, t + 1))
    return M


def test_channel_constant_gate_is_forgetting_attention():
    rng = np.random.default_rng(12)
    T, H, D = 29, 2, 6
    q, k, v, _, w, _ = make(rng, 1, T, H, H, D, D)
    a = -np.log1p(np.exp(-(rnd(rng, T, H) + 1.0)))             # scalar gate per (t, head)
    g = np.repeat(a[None, :, :, None], D, axis=3)
    scale = D ** -0.5
    out = fix_ref.forward(q, k, v, g, w, None, scale, 0.0)
    for h in range(H):
        M = _fox_mask(a[:, h])
        sd = _sdpa(q[0, :, h:h + 1], k[0, :, h:h + 1], v[0, :, h:h + 1], M[None], scale)[:, 0]
        assert relerr(out["y"][0, :, h], _rms(sd, w, 0.0)) < 1e-12


def test_each_channel_is_forgetting_attention_with_its_own_gate():
    # pins the element-wise decay channel by channel (o before the norm)
    rng = np.random.default_rng(13)
    T, D = 23, 5
    q, k, v, g, w, _ = make(rng, 1, T, 1, 1, 4, D)
    scale = 0.5
    out = fix_ref.forward(q, k, v, g, w, None, scale, 1e-6)
    S = scale * q[0, :, 0] @ k[0, :, 0].T
    Sm = np.where(np.tri(T, dtype=bool), S, -np.inf)
    m = Sm.max(-1)
    for c in range(D):
        M = _fox_mask(g[0, :, 0, c])
        sd = _sdpa(q[0, :, :1], k[0, :, :1], v[0, :, :1, c:c + 1], M[None], scale)[:, 0, 0]
        ell = np.exp(Sm + M - m[:, None]).sum(-1)
        assert relerr(out["o"][0, :, 0, c], sd * ell) < 1e-12


# ----------------------------------------------------------- closed forms

def test_golden_two_token_example():
    path = os.path.join(HERE, "golden", "fix_two_token_example.txt")
    text = "".join(l for l in open(path) if not l.lstrip().startswith("#"))
    ex = json.loads(text)
    arr = lambda key: np.array(ex[key], np.float64)[None]
    out = fix_ref.forward(arr("q"), arr("k"), arr("v"), arr("g"), np.array(ex["w"]),
                          None, ex["scale"], ex["eps"])
    e1 = math.exp(-1.0)
    y0 = np.array([2.0, 4.0]) / math.sqrt(10.0)
    y1 = np.array([1 + e1, 1 - e1]) / math.sqrt(1 + e1 * e1)
    assert np.allclose(out["y"][0, 0, 0], y0, rtol=0, atol=1e-14)
    assert np.allclose(out["y"][0, 1, 0], y1, rtol=0, atol=1e-14)
    assert np.allclose(out["m"][0, :, 0], [0.5, 1.0], rtol=0, atol=1e-15)


def test_length_one_sequence_is_rmsnorm_of_v():
    rng = np.random.default_rng(14)
    q, k, v, g, w, _ = make(rng, 3, 1, 4, 2, 8, 8)
    eps = 1e-6
    out = fix_ref.forward(q, k, v, g, w, None, None, eps)
    vr = np.repeat(v, 2, axis=2)
    assert relerr(out["y"], _rms(vr, w, eps)) < 1e-14
    # every length-1 sequence of a packed batch, too
    q, k, v, g, w, _ = make(rng, 1, 5, 2, 1, 4, 4)
    out = fix_ref.forward(q, k, v, g, w, [1, 1, 1, 1, 1], None, eps)
    assert relerr(out["y"], _rms(np.repeat(v, 2, axis=2), w, eps)) < 1e-14


def test_total_forgetting_keeps_only_the_diagonal():
    rng = np.random.default_rng(15)
    q, k, v, _, w, _ = make(rng, 1, 9, 2, 2, 4, 4)
    g = np.full(v.shape, -1e4)
    out = fix_ref.forward(q, k, v, g, w, None, 0.5, 0.0)
    assert relerr(out["y"], _rms(v, w, 0.0)) < 1e-13


def test_value_scale_invariance_at_eps0():
    rng = np.random.default_rng(16)
    q, k, v, g, w, _ = make(rng, 1, 12, 2, 1, 4, 4)
    a = fix_ref.forward(q, k, v, g, w, None, None, 0.0)["y"]
    b = fix_ref.forward(q, k, 3.7 * v, g, w, None, None, 0.0)["y"]
    assert relerr(a, b) < 1e-13


# ----------------------------------------------------------- invariants

def test_first_gate_of_each_sequence_is_unused():
    rng = np.random.default_rng(17)
    q, k, v, g, w, dy = make(rng, 1, 10, 2, 1, 4, 4)
    seqlens = [4, 6]
    a = fix_ref.forward(q, k, v, g, w, seqlens)["y"]
    g2 = g.copy(); g2[0, 0] += 5.0; g2[0, 4] -= 3.0
    b = fix_ref.forward(q, k, v, g2, w, seqlens)["y"]
    assert np.array_equal(a, b) or relerr(a, b) < 1e-15
    grads = fix_ref.backward(q, k, v, g, w, dy, seqlens)
    assert np.abs(grads["dg"][0, [0, 4]]).max() < 1e-12 * np.abs(grads["dg"]).max()


def test_dG_identity_and_zero_sum():
    # dG_t = sum_h do_t * o_t - v_t * dv_t (the block-friendly form) equals the
    # per-pair form the oracle uses; shift invariance of G gives sum_t dG_t = 0
    rng = np.random.default_rng(18)
    q, k, v, g, w, dy = make(rng, 1, 11, 2, 1, 3, 4)
    scale, eps = 0.6, 1e-6
    grads = fix_ref.backward(q, k, v, g, w, dy, None, scale, eps)
    out = fix_ref.forward(q, k, v, g, w, None, scale, eps)
    n = out["o"] * out["rstd"][..., None]
    dn = dy * w
    do = out["rstd"][..., None] * (dn - n * (dn * n).mean(-1, keepdims=True))
    A = (do * out["o"]).sum(axis=2)                              # over the 2 q heads
    dG = A - v[:, :, 0] * grads["dv"][:, :, 0]
    dg = np.cumsum(dG[:, ::-1], axis=1)[:, ::-1]
    assert relerr(grads["dg"][:, :, 0], dg) < 1e-12
    assert abs(dG.sum(axis=1)).max() < 1e-12 * abs(dG).max()


def test_varlen_equals_independent_sequences():
    rng = np.random.default_rng(19)
    seqlens = [5, 0, 9, 1, 3]
    T = sum(seqlens)
    q, k, v, g, w, dy = make(rng, 1, T, 4, 2, 4, 4)
    f = fix_ref.forward(q, k, v, g, w, seqlens)
    gr = fix_ref.backward(q, k, v, g, w, dy, seqlens)
    s0 = 0
    for L in seqlens:
        sl = slice(s0, s0 + L)
        f1 = fix_ref.forward(q[:, sl], k[:, sl], v[:, sl], g[:, sl], w)
        g1 = fix_ref.backward(q[:, sl], k[:, sl], v[:, sl], g[:, sl], w, dy[:, sl])
        if L:
            assert relerr(f["y"][:, sl], f1["y"]) < 1e-14
            for key in ("dq", "dk", "dv", "dg"):
                assert relerr(gr[key][:, sl], g1[key]) < 1e-13
        s0 += L


def test_gqa_equals_mha_with_repeated_kv():
    rng = np.random.default_rng(20)
    q, k, v, g, w, dy = make(rng, 2, 7, 6, 2, 4, 4)
    a = fix_ref.forward(q, k, v, g, w)
    ga = fix_ref.backward(q, k, v, g, w, dy)
    kr, vr, gr_ = (np.repeat(x, 3, axis=2) for x in (k, v, g))
    b = fix_ref.forward(q, kr, vr, gr_, w)
    gb = fix_ref.backward(q, kr, vr, gr_, w, dy)
    assert relerr(a["y"], b["y"]) < 1e-14
    assert relerr(ga["dq"], gb["dq"]) < 1e-13
    for key in ("dk", "dv", "dg"):
        summed = gb[key].reshape(2, 7, 2, 3, 4).sum(axis=3)
        assert relerr(ga[key], summed) < 1e-13


# ----------------------------------------------------- sampled-output helpers

def test_row_helpers_match_full_oracle():
    rng = np.random.default_rng(21)
    seqlens = [9, 14]
    q, k, v, g, w, dy = make(rng, 1, 23, 4, 2, 4, 4)
    full = fix_ref.forward(q, k, v, g, w, seqlens)
    grads = fix_ref.backward(q, k, v, g, w, dy, seqlens)
    start, L, h = 9, 14, 3
    rows = [0, 5, 13]
    r = fix_ref.forward_rows(q, k, v, g, w, start, L, h, rows)
    assert relerr(r["y"], full["y"][0, [start + t for t in rows], h]) < 1e-14
    dq = fix_ref.dq_rows(q, k, v, g, w, dy, start, L, h, rows)
    assert relerr(dq, grads["dq"][0, [start + t for t in rows], h]) < 1e-13
    R = 6
    sb = fix_ref.suffix_backward(q, k, v, g, w, dy, start, L, 1, R)
    sl = slice(start + L - R, start + L)
    for key in ("dk", "dv", "dg"):
        assert relerr(sb[key], grads[key][0, sl, 1]) < 1e-12, key


def test_process_pool_equals_serial():
    """The GPU parity tests run the oracle over a spawn process pool
    (workers > 1); its results must be bit-identical to the serial branch,
    which the pins above check.  Each (sequence, head) unit is computed by the
    same function either way, so any difference would come from the pool's
    job bookkeeping (a unit written to the wrong place, a group sum taken
    twice or missed)."""
    rng = np.random.default_rng(17)
    q, k, v, g, w, dy = make(rng, 1, 23, 4, 2, 4, 4)
    seqlens = [5, 0, 11, 7]
    serial_f = fix_ref.forward(q, k, v, g, w, seqlens, None, 1e-6, workers=1)
    pool_f = fix_ref.forward(q, k, v, g, w, seqlens, None, 1e-6, workers=2)
    serial_b = fix_ref.backward(q, k, v, g, w, dy, seqlens, None, 1e-6, workers=1)
    pool_b = fix_ref.backward(q, k, v, g, w, dy, seqlens, None, 1e-6, workers=2)
    for key in serial_f:
        assert np.array_equal(serial_f[key], pool_f[key]), key
    for key in serial_b:
        assert np.array_equal(serial_b[key], pool_b[key]), key
    # batched (B > 1) problems take the same path
    q, k, v, g, w, dy = make(rng, 3, 9, 2, 1, 4, 2)
    a = fix_ref.backward(q, k, v, g, w, dy, None, None, 1e-6, workers=1)
    b = fix_ref.backward(q, k, v, g, w, dy, None, None, 1e-6, workers=3)
    for key in a:
        assert np.array_equal(a[key], b[key]), key


# ----------------------------------------- o_gate, o_norm = False, scalar gate
# FiX README "Quick Start": o_norm, o_norm_weight and o_gate are arguments of
# the same call; the Forgetting Transformer abstract: scalar forget gates.

def test_output_gate_is_swish_after_norm_and_weight():
    """y with o_gate z equals y without it times torch's silu(z) = z sigmoid(z),
    element by element, with and without the RMSNorm."""
    rng = np.random.default_rng(31)
    q, k, v, g, w, _ = make(rng, 2, 9, 4, 2, 4, 6)
    z = 2.0 * rnd(rng, 2, 9, 4, 6)
    silu = torch.nn.functional.silu(torch.from_numpy(z)).numpy()
    for norm in (True, False):
        a = fix_ref.forward(q, k, v, g, w, None, 0.6, 1e-6, norm=norm)["y"]
        b = fix_ref.forward(q, k, v, g, w, None, 0.6, 1e-6, norm=norm, o_gate=z)["y"]
        assert relerr(b, a * silu) < 1e-14


def test_no_norm_zero_gate_is_causal_softmax_attention():
    """o_norm = False with g = 0 is ordinary causal softmax attention (torch
    SDPA), whatever eps, and does not depend on the row shift."""
    rng = np.random.default_rng(32)
    T, Hq, Hkv, D = 31, 4, 2, 8
    q, k, v, _, w, _ = make(rng, 1, T, Hq, Hkv, D, D)
    g = np.zeros((1, T, Hkv, D))
    kr, vr = np.repeat(k[0], 2, axis=1), np.repeat(v[0], 2, axis=1)
    sd = _sdpa(q[0], kr, vr, scale=0.3)
    y = fix_ref.forward(q, k, v, g, w, None, 0.3, 1e-3, norm=False)["y"][0]
    assert relerr(y, sd) < 1e-13


def test_no_norm_closed_forms():
    rng = np.random.default_rng(33)
    # T = 1: the output is v_0
    q, k, v, g, w, _ = make(rng, 2, 1, 2, 1, 4, 4)
    y = fix_ref.forward(q, k, v, g, w, None, None, 1e-6, norm=False)["y"]
    assert relerr(y, np.repeat(v, 2, axis=2)) < 1e-15
    # total forgetting: o_t = softmax_t(S)[t] v_t
    T = 7
    q, k, v, _, w, _ = make(rng, 1, T, 1, 1, 3, 3)
    g = np.full(v.shape, -1e4)
    y = fix_ref.forward(q, k, v, g, w, None, 0.5, 0.0, norm=False)["y"][0, :, 0]
    S = 0.5 * q[0, :, 0] @ k[0, :, 0].T
    Sm = np.where(np.tri(T, dtype=bool), S, -np.inf)
    p = np.exp(Sm - Sm.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    assert relerr(y, np.diag(p)[:, None] * v[0, :, 0]) < 1e-13


def _fd_variant(norm, gated, scalar, seed):
    rng = np.random.default_rng(seed)
    B, T, Hq, Hkv, Dk, Dv = 1, 5, 2, 1, 3, 3
    q, k, v, g, w, dy = make(rng, B, T, Hq, Hkv, Dk, Dv)
    if scalar:
        g = g[..., 0].copy()
    z = rnd(rng, B, T, Hq, Dv) if gated else None
    scale, eps = 0.8, 1e-2
    grads = fix_ref.backward(q, k, v, g, w, dy, None, scale, eps, norm=norm, o_gate=z)
    m0 = fix_ref.forward(q, k, v, g, w, None, scale, eps)["m"]
    args = dict(q=q, k=k, v=v, g=g, w=w)
    names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("w", "dw")]
    if gated:
        args["z"] = z
        names.append(("z", "d_o_gate"))
    h = 1e-5
    for name, gname in names:
        x = args[name]
        fd = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            old = x[idx]
            x[idx] = old + h
            # norm = False: the output does not depend on m at all, so m free
            lp = brute_loss(q, k, v, g, w, dy, None, scale, eps, m0 if norm else None, norm, z)
            x[idx] = old - h
            lm = brute_loss(q, k, v, g, w, dy, None, scale, eps, m0 if norm else None, norm, z)
            x[idx] = old
            fd[idx] = (lp - lm) / (2 * h)
        assert grads[gname].shape == x.shape, gname
        err = relerr(grads[gname], fd)
        assert err < 1e-7 or np.abs(fd).max() < 1e-12, (name, err)


@pytest.mark.parametrize("norm,gated,scalar", [
    (True, True, False), (False, False, False), (False, True, False),
    (True, False, True), (False, True, True),
])
def test_variant_gradients_match_finite_differences(norm, gated, scalar):
    _fd_variant(norm, gated, scalar, seed=34)


def test_scalar_gate_is_the_channel_broadcast_and_forgetting_attention():
    """A gate [B,T,Hkv] is the element-wise gate broadcast over channels; at
    eps = 0 that is RMSNorm of Forgetting-Transformer attention (SDPA with the
    additive bias G_t - G_s); its dg is the channel sum."""
    rng = np.random.default_rng(35)
    T, H, D = 21, 2, 5
    q, k, v, _, w, dy = make(rng, 1, T, H, H, D, D)
    a = -np.log1p(np.exp(-(rnd(rng, 1, T, H) + 1.0)))
    gb = np.repeat(a[..., None], D, axis=3)
    ys = fix_ref.forward(q, k, v, a, w, None, 0.4, 0.0)["y"]
    yb = fix_ref.forward(q, k, v, gb, w, None, 0.4, 0.0)["y"]
    assert np.array_equal(ys, yb)
    for h in range(H):
        M = _fox_mask(a[0, :, h])
        sd = _sdpa(q[0, :, h:h + 1], k[0, :, h:h + 1], v[0, :, h:h + 1], M[None], 0.4)[:, 0]
        assert relerr(ys[0, :, h], _rms(sd, w, 0.0)) < 1e-12
    gs = fix_ref.backward(q, k, v, a, w, dy, None, 0.4, 1e-6)
    gbr = fix_ref.backward(q, k, v, gb, w, dy, None, 0.4, 1e-6)
    assert gs["dg"].shape == a.shape
    assert relerr(gs["dg"], gbr["dg"].sum(axis=-1)) < 1e-14

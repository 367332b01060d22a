"""The oracle's pins must catch plausible mistakes.

Each case plants one slip in a private copy of the oracle's source (on the
CPU; the real module is untouched) and checks that the brute-force or
finite-difference pin rejects the mutated oracle.
"""
import inspect
import types

import numpy as np
import pytest

from oracle import brute_forward, brute_loss, fix_ref

SRC = inspect.getsource(fix_ref)

MUTATIONS = {
    # decay summed over r in [s, t] instead of (s, t]
    "decay_includes_s": ("D = np.exp(G[t][None, :] - G[: t + 1])     # D_ts[c], s = 0..t",
                         "D = np.exp(G[t][None, :] - G[: t + 1] + g[: t + 1])"),
    # RMSNorm without eps
    "rms_drops_eps": ("rstd = 1.0 / np.sqrt((o * o).mean(axis=1) + eps)",
                      "rstd = 1.0 / np.sqrt((o * o).mean(axis=1))"),
    # wrong sign of the gate gradient's key-side term
    "dG_sign": ("dG[: t + 1] -= W * do[t][None, :] * V[: t + 1]",
                "dG[: t + 1] += W * do[t][None, :] * V[: t + 1]"),
    # transposed dS in dK
    "dK_transposed": ("dK = scale * (dS.T @ Q)", "dK = scale * (dS @ Q)"),
    # RMSNorm backward without its projection term
    "do_missing_mean": ("do = rstd[:, None] * (dn - n * (dn * n).mean(axis=1, keepdims=True))",
                        "do = rstd[:, None] * dn"),
    # forward instead of reverse cumsum for dg
    "dg_forward_cumsum": ("dg = np.cumsum(dG[::-1], axis=0)[::-1]         # dg_r = sum_{t>=r} dG_t",
                          "dg = np.cumsum(dG, axis=0)"),
    # GQA: q head h mapped to kv head h % Hkv instead of h // group
    "gqa_modulo": ("kv = h // grp\n            sl = slice(s0, s0 + L)\n            jobs.append((q[b, sl, h], k[b, sl, kv], v[b, sl, kv], g[b, sl, kv], w, scale, eps))",
                   "kv = h % Hkv\n            sl = slice(s0, s0 + L)\n            jobs.append((q[b, sl, h], k[b, sl, kv], v[b, sl, kv], g[b, sl, kv], w, scale, eps))"),
    # output gate applied as sigmoid(z) instead of z * sigmoid(z)
    "gate_sigmoid_only": ("    return z / (1.0 + np.exp(-z))", "    return 1.0 / (1.0 + np.exp(-z))"),
    # swish derivative without its second term
    "gate_grad_drops_term": ("    return sg * (1.0 + z * (1.0 - sg))", "    return sg"),
    # no-norm backward without the softmax-denominator term
    "nonorm_drops_delta": ("        dS = P * (dP - (do * o).sum(axis=1)[:, None])",
                           "        dS = P * dP"),
    # no-norm output divided by the row maximum's weight instead of the sum
    "nonorm_wrong_denominator": ("        y = o / P.sum(axis=1)[:, None]             # softmax denominator l_t",
                                 "        y = o / P.max(axis=1)[:, None]"),
}


def mutated(name):
    old, new = MUTATIONS[name]
    assert SRC.count(old) >= 1, name
    mod = types.ModuleType("fix_ref_mut_" + name)
    exec(compile(SRC.replace(old, new, 1), mod.__name__, "exec"), mod.__dict__)
    return mod


def _inputs(seed=1, T=5, Hq=2, Hkv=1, D=3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, T, Hq, D)); k = rng.standard_normal((1, T, Hkv, D))
    v = rng.standard_normal((1, T, Hkv, D))
    g = -np.log1p(np.exp(-(rng.standard_normal((1, T, Hkv, D)) + 1)))
    w = 1 + 0.1 * rng.standard_normal(D); dy = rng.standard_normal((1, T, Hq, D))
    return q, k, v, g, w, dy


VARIANTS = [dict(norm=True, gated=False), dict(norm=True, gated=True),
            dict(norm=False, gated=False), dict(norm=False, gated=True)]


def _gate(seed, q):
    return np.random.default_rng(seed + 100).standard_normal(q.shape[:3] + (3,))


def _forward_pin_fails(mod):
    q, k, v, g, w, _ = _inputs(Hq=4, Hkv=2)
    for var in VARIANTS:
        z = _gate(1, q) if var["gated"] else None
        y = mod.forward(q, k, v, g, w, None, 0.7, 1e-2, norm=var["norm"], o_gate=z)["y"]
        yb, _ = brute_forward(q, k, v, g, w, None, 0.7, 1e-2, None, var["norm"], z)
        if not np.allclose(y, np.array(yb), rtol=1e-10, atol=1e-12):
            return True
    return False


def _fd_pin_fails(mod):
    q, k, v, g, w, dy = _inputs()
    scale, eps = 0.8, 1e-2
    for var in VARIANTS:
        z = _gate(2, q) if var["gated"] else None
        gr = mod.backward(q, k, v, g, w, dy, None, scale, eps, norm=var["norm"], o_gate=z)
        m0 = fix_ref.forward(q, k, v, g, w, None, scale, eps)["m"]
        args = dict(q=q, k=k, v=v, g=g, w=w)
        names = [("q", "dq"), ("k", "dk"), ("v", "dv"), ("g", "dg"), ("w", "dw")]
        if z is not None:
            args["z"] = z
            names.append(("z", "d_o_gate"))
        for name, gname in names:
            x = args[name]
            fd = np.zeros_like(x)
            for idx in np.ndindex(x.shape):
                old = x[idx]
                x[idx] = old + 1e-5
                lp = brute_loss(q, k, v, g, w, dy, None, scale, eps, m0, var["norm"], z)
                x[idx] = old - 1e-5
                lm = brute_loss(q, k, v, g, w, dy, None, scale, eps, m0, var["norm"], z)
                x[idx] = old
                fd[idx] = (lp - lm) / 2e-5
            if not np.allclose(gr[gname], fd, rtol=1e-6, atol=1e-8):
                return True
    return False


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_reject_planted_mistake(name):
    mod = mutated(name)
    assert _forward_pin_fails(mod) or _fd_pin_fails(mod), f"mutation {name} not caught"


def test_unmutated_oracle_passes_same_checks():
    assert not _forward_pin_fails(fix_ref)
    assert not _fd_pin_fails(fix_ref)

"""Host-side checks of the C ABI (no GPU needed, no kernel is launched).

The library must load, export every function that include/fix_attn.h
declares, size its workspace, and reject bad arguments on the host with the
documented status codes before touching the device.
"""
import ctypes
import os
import re

import pytest
import torch

from gated_softmax_attention_fp32_b200 import fixattn

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fix_attn.h")

FIX_OK, FIX_ERR_NULL, FIX_ERR_SHAPE, FIX_ERR_HEAD_DIM, FIX_ERR_GQA = 0, 1, 2, 3, 4
FIX_ERR_CU_SEQLENS, FIX_ERR_ALIGN, FIX_ERR_WORKSPACE, FIX_ERR_DTYPE = 5, 6, 7, 8


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fix_attn_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from gated_softmax_attention_fp32_b200 import build
    if not os.path.exists(fixattn.LIB_PATH):
        build.build()
    return fixattn.load()


def test_library_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) >= {"fix_attn_fwd", "fix_attn_bwd", "fix_attn_workspace_bytes",
                          "fix_attn_device_status", "fix_attn_status_string"}
    raw = ctypes.CDLL(fixattn.LIB_PATH)
    for n in names:
        assert hasattr(raw, n), n
    # the binding names every declared entry point, and nothing else
    assert set(names) == set(fixattn.EXPORTS)


def prob(B=2, T=100, Hq=4, Hkv=2, Dk=64, Dv=64, **kw):
    p = fixattn.Problem()
    p.batch, p.seqlen, p.num_q_heads, p.num_kv_heads = B, T, Hq, Hkv
    p.head_dim_k, p.head_dim_v = Dk, Dv
    p.num_seqs = 0
    p.y_dtype = 0
    p.algo = 0
    p.flags = 0
    p.scale = 0.0
    p.eps = 1e-6
    for key, val in kw.items():
        setattr(p, key, val)
    return p


def test_workspace_sizes(lib):
    ws_f = lib.fix_attn_workspace_bytes(ctypes.byref(prob()), 0)
    ws_b = lib.fix_attn_workspace_bytes(ctypes.byref(prob()), 1)
    assert 0 < ws_f < ws_b
    # L (f32) + pre-decayed v (bf16) dominate the forward workspace
    assert ws_f >= 2 * 100 * 2 * 64 * 6
    assert lib.fix_attn_workspace_bytes(ctypes.byref(prob(Dk=48)), 0) == 0
    assert lib.fix_attn_workspace_bytes(None, 0) == 0


def _ceil(a, b):
    return -(-a // b)


def _expected_workspace(seqlens, Hq, Hkv, Dk, Dv, backward):
    """The workspace layout written out from its documented parts: 256-byte
    aligned buffers, and for the backward the dk/dv split (per key chunk, its
    diagonal tiles and its later tiles, each cut into runs of at most P tiles,
    P sized for about one run per SM of a 148-SM B200), one partial slot of
    128 rows x (Dk + Dv) floats per run and kv head."""
    grp = Hq // Hkv
    N = sum(seqlens)
    nchunks = sum(_ceil(L, 128) for L in seqlens)
    nc1 = max(nchunks, 1)
    o = 0

    def take(nbytes):
        nonlocal o
        o = _ceil(o + nbytes, 256) * 256

    nkv, nch = N * Hkv * Dv, nchunks * Hkv * Dv
    # status, chunk table, order, safe flags, L and its channel-major copy,
    # Vt, Vm hi, Vm lo, then the per-(chunk, kv head, channel) tot, rho, hr
    # and log2 max |Vt|
    for nbytes in (256, nc1 * 16, nc1 * 4, nc1 * Hkv * 4, nkv * 4, nkv * 4, nkv * 2, nkv * 2,
                   nkv * 2, nch * 4, nch * 4, nch * 4, nch * 4):
        take(nbytes)
    if not backward:
        return o
    t64 = lambda L, j: (L - 128 * j + 63) // 64          # query tiles from chunk j on
    half = lambda L, j: (min(128, L - 128 * j) + 63) // 64
    total = Hkv * sum(grp * t64(L, j) for L in seqlens for j in range(_ceil(L, 128)))
    P = max(4, _ceil(total, 148))
    nparts = sum(_ceil(grp * half(L, j), P) + _ceil(grp * (t64(L, j) - half(L, j)), P)
                 for L in seqlens for j in range(_ceil(L, 128)))
    for nbytes in (N * Hq * Dv * 4, N * Hq * Dv * 2, N * Hq * Dv * 2, N * Hq * Dv * 2,
                   nc1 * Hq * 4, nc1 * Hq * 4, N * Hq * 4, N * Hq * 4, nkv * 4, nkv * 4, nch * 4,
                   nc1 * 2 * Hkv * Dv * 4, max(nparts, 1) * 16, nc1 * 8,
                   nparts * Hkv * 128 * (Dk + Dv) * 4):
        take(nbytes)
    return o


@pytest.mark.parametrize("seqlens,Hq,Hkv,Dk,Dv", [
    ([2048, 2048], 8, 4, 128, 128),
    ([100, 100], 4, 2, 64, 64),
    ([2817, 6892, 6576, 99], 16, 4, 128, 128),
    ([0, 1, 130, 7, 255, 0, 64, 300], 4, 2, 64, 128),
    ([4096] * 8, 16, 16, 64, 64),
    ([129, 640], 32, 2, 128, 64),
])
def test_workspace_layout_and_dkv_split(lib, seqlens, Hq, Hkv, Dk, Dv):
    """Sizes the workspace (and so the dk/dv work split it holds slots for)
    the way the host plans it, for fixed-length and packed problems."""
    if len(set(seqlens)) == 1:
        p = prob(B=len(seqlens), T=seqlens[0], Hq=Hq, Hkv=Hkv, Dk=Dk, Dv=Dv)
        keep = None
    else:
        cu = [0]
        for L in seqlens:
            cu.append(cu[-1] + L)
        keep = (ctypes.c_int64 * len(cu))(*cu)
        p = prob(B=1, T=cu[-1], Hq=Hq, Hkv=Hkv, Dk=Dk, Dv=Dv, num_seqs=len(seqlens),
                 cu_seqlens_host=ctypes.addressof(keep), cu_seqlens=ctypes.addressof(keep))
    for backward in (0, 1):
        got = lib.fix_attn_workspace_bytes(ctypes.byref(p), backward)
        assert got == _expected_workspace(seqlens, Hq, Hkv, Dk, Dv, backward), (backward, got)
    del keep


@pytest.mark.parametrize("kw,code", [
    (dict(Dk=48), FIX_ERR_HEAD_DIM),
    (dict(Dv=256), FIX_ERR_HEAD_DIM),
    (dict(Hq=6, Hkv=4), FIX_ERR_GQA),
    (dict(B=0), FIX_ERR_SHAPE),
    (dict(T=-1), FIX_ERR_SHAPE),
    (dict(y_dtype=7), FIX_ERR_DTYPE),
    (dict(algo=9), FIX_ERR_DTYPE),
    (dict(flags=8), FIX_ERR_SHAPE),
    (dict(eps=-1.0), FIX_ERR_SHAPE),
    (dict(num_seqs=2), FIX_ERR_CU_SEQLENS),
])
def test_bad_problem_rejected_on_host(lib, kw, code):
    p = prob(**kw)
    buf = (ctypes.c_uint8 * 4096)()
    a = ctypes.addressof(buf)
    a = (a + 15) // 16 * 16
    ptrs = [ctypes.c_void_p(a)] * 11
    s = lib.fix_attn_fwd(ctypes.byref(p), *ptrs, 1 << 40, None)
    assert s == code, fixattn.status_string(s)
    ptrs = [ctypes.c_void_p(a)] * 17
    s = lib.fix_attn_bwd(ctypes.byref(p), *ptrs, 1 << 40, None)
    assert s == code, fixattn.status_string(s)


def _cu_problem(cu):
    host = torch.tensor(cu, dtype=torch.int64)
    p = prob(B=1, T=int(cu[-1]) if cu else 0, num_seqs=len(cu) - 1)
    p.cu_seqlens = host.data_ptr()          # any non-NULL pointer: never dereferenced here
    p.cu_seqlens_host = host.data_ptr()
    return p, host


@pytest.mark.parametrize("cu,code", [
    ([1, 5, 10], FIX_ERR_CU_SEQLENS),
    ([0, 5, 3, 10], FIX_ERR_CU_SEQLENS),
])
def test_bad_cu_seqlens_rejected(lib, cu, code):
    p, host = _cu_problem(cu)
    p.seqlen = 10
    assert lib.fix_attn_workspace_bytes(ctypes.byref(p), 0) == 0
    buf = (ctypes.c_uint8 * 64)()
    a = (ctypes.addressof(buf) + 15) // 16 * 16
    s = lib.fix_attn_fwd(ctypes.byref(p), *[ctypes.c_void_p(a)] * 11, 1 << 40, None)
    assert s == code


def test_varlen_requires_batch_one_and_host_mirror(lib):
    p, host = _cu_problem([0, 4, 10])
    p.batch = 2
    p.seqlen = 5
    assert lib.fix_attn_workspace_bytes(ctypes.byref(p), 0) == 0
    p, host = _cu_problem([0, 4, 10])
    p.cu_seqlens_host = None
    assert lib.fix_attn_workspace_bytes(ctypes.byref(p), 0) == 0
    p, host = _cu_problem([0, 0, 4, 4, 10])       # empty sequences are legal
    assert lib.fix_attn_workspace_bytes(ctypes.byref(p), 1) > 0


def test_null_misaligned_and_small_workspace(lib):
    p = prob()
    need = lib.fix_attn_workspace_bytes(ctypes.byref(p), 0)
    buf = (ctypes.c_uint8 * 4096)()
    a = (ctypes.addressof(buf) + 15) // 16 * 16
    # q, k, v, g, w, o_gate, y, o_saved, m_saved, rstd_saved, workspace
    good = [ctypes.c_void_p(a)] * 11
    s = lib.fix_attn_fwd(ctypes.byref(p), *([None] + good[1:]), need, None)
    assert s == FIX_ERR_NULL
    bad = list(good)
    bad[2] = ctypes.c_void_p(a + 2)
    assert lib.fix_attn_fwd(ctypes.byref(p), *bad, need, None) == FIX_ERR_ALIGN
    bad = list(good)
    bad[5] = ctypes.c_void_p(a + 4)                 # a misaligned output gate
    assert lib.fix_attn_fwd(ctypes.byref(p), *bad, need, None) == FIX_ERR_ALIGN
    assert lib.fix_attn_fwd(ctypes.byref(p), *good, need - 1, None) == FIX_ERR_WORKSPACE
    # saved tensors: all three or none
    part = list(good)
    part[8] = None
    assert lib.fix_attn_fwd(ctypes.byref(p), *part, need, None) == FIX_ERR_NULL
    # o_norm_weight is required with the norm, optional without it
    now = list(good)
    now[4] = None
    assert lib.fix_attn_fwd(ctypes.byref(p), *now, need, None) == FIX_ERR_NULL
    # backward: o_gate and d_o_gate both given or both NULL
    pb = prob()
    needb = lib.fix_attn_workspace_bytes(ctypes.byref(pb), 1)
    gb = [ctypes.c_void_p(a)] * 17
    half = list(gb)
    half[16] = None                                  # d_o_gate missing, o_gate given
    assert lib.fix_attn_bwd(ctypes.byref(pb), *half, needb, None) == FIX_ERR_NULL


def test_flag_dependent_workspace(lib):
    """Without the norm the forward workspace is the same; a scalar gate adds
    the per-channel dg buffer to the backward's."""
    base0 = lib.fix_attn_workspace_bytes(ctypes.byref(prob()), 0)
    base1 = lib.fix_attn_workspace_bytes(ctypes.byref(prob()), 1)
    assert lib.fix_attn_workspace_bytes(ctypes.byref(prob(flags=2)), 0) == base0
    assert lib.fix_attn_workspace_bytes(ctypes.byref(prob(flags=2)), 1) == base1
    assert lib.fix_attn_workspace_bytes(ctypes.byref(prob(flags=4)), 0) == base0
    extra = lib.fix_attn_workspace_bytes(ctypes.byref(prob(flags=4)), 1) - base1
    assert extra == -(-(2 * 100 * 2 * 64 * 4) // 256) * 256


def test_status_strings(lib):
    for c in range(12):
        s = fixattn.status_string(c)
        assert s.startswith("FIX_")
    assert "unknown" in fixattn.status_string(99)


def test_missing_library_fails_loudly(tmp_path):
    """No fallback on the product path: without the CUDA library every call
    raises instead of computing anything another way."""
    import subprocess
    import sys
    code = (
        "import sys; sys.path.insert(0, %r)\n"
        "from gated_softmax_attention_fp32_b200 import fixattn\n"
        "fixattn.LIB_PATH = %r\n"
        "try:\n"
        "    fixattn.load()\n"
        "except RuntimeError as e:\n"
        "    print('raised:', e)\n"
        "    sys.exit(0)\n"
        "sys.exit(1)\n" % (ROOT, str(tmp_path / "absent.so")))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and "not built" in r.stdout, r.stdout + r.stderr

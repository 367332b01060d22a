"""fix_attn_fwd_noalloc: the forward for callers that cannot allocate.

Some callers have no device allocator at hand when they call the forward
(host code given only tensors and a stream, or a runtime whose device memory
is fixed up front).  fix_attn_fwd_noalloc serves them from a fixed device
array inside the library.  These tests call it through the C ABI and check
that two calls in a row (different inputs, so nothing stale from the first
call may leak into the second) give the forward of the ordinary entry point,
within the parity tolerance the other tests use.  This file is collected
last so that a failure here stops a run only after every other test ran.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from fixtools import FWD_MAX_ABS, FWD_REL_L2, max_abs, rel_l2

pytestmark = pytest.mark.gpu

FIX_ERR_WORKSPACE = 7


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc_call(lib, fixattn, t, cu=None, cu_host=None):
    """Raw C-ABI call; outputs start as NaN so every element must be written."""
    B, T, Hq, _ = t["q"].shape
    Dv = t["v"].shape[3]
    p, keep = fixattn.make_problem(t["q"], t["k"], t["v"], cu, cu_host, None, 1e-6,
                                   torch.float32)
    y = torch.full((B, T, Hq, Dv), float("nan"), device="cuda")
    o = torch.full((B, T, Hq, Dv), float("nan"), device="cuda")
    m = torch.full((B, T, Hq), float("nan"), device="cuda")
    r = torch.full((B, T, Hq), float("nan"), device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    s = lib.fix_attn_fwd_noalloc(ctypes.byref(p), _ptr(t["q"]), _ptr(t["k"]), _ptr(t["v"]),
                                 _ptr(t["g"]), _ptr(t["w"]), _ptr(y), _ptr(o), _ptr(m), _ptr(r),
                                 stream)
    torch.cuda.synchronize()
    del keep
    return s, y, (o, m, r)


def _inputs(seed, seqlens=None, B=2, T=300):
    case = synth.make_case(B, T, 4, 2, 64, 64, seed=seed, seqlens=seqlens)
    t = {k: case[k].cuda().contiguous() for k in ("q", "k", "v", "g", "w")}
    cu = case["cu_seqlens"]
    return t, (cu.cuda() if cu is not None else None), cu


def test_noalloc_forward_matches_workspace_forward_two_calls(cuda_lib):
    from gated_softmax_attention_fp32_b200 import fixattn
    lib = fixattn.load()
    for seed, seqlens in ((11, None), (12, [5, 0, 260, 1, 140])):
        t, cu, cu_host = _inputs(seed, seqlens, B=1 if seqlens else 2)
        s, y, saved = _noalloc_call(lib, fixattn, t, cu, cu_host)
        assert s == 0, fixattn.status_string(s)
        y_ref, saved_ref = fixattn.fix_attn_fwd(t["q"], t["k"], t["v"], t["g"], t["w"], cu,
                                                cu_host, y_dtype=torch.float32)
        torch.cuda.synchronize()
        a, b = y.double().cpu().numpy(), y_ref.double().cpu().numpy()
        assert np.isfinite(a).all()
        assert rel_l2(a, b) <= FWD_REL_L2 and max_abs(a, b) <= FWD_MAX_ABS
        for x, xr in zip(saved, saved_ref):
            assert rel_l2(x.double().cpu().numpy(), xr.double().cpu().numpy()) <= FWD_REL_L2


def test_noalloc_rejects_problem_beyond_its_workspace(cuda_lib):
    from gated_softmax_attention_fp32_b200 import fixattn
    lib = fixattn.load()
    p = fixattn.Problem()
    p.batch, p.seqlen, p.num_q_heads, p.num_kv_heads = 1, 1 << 16, 8, 8
    p.head_dim_k = p.head_dim_v = 128
    p.eps = 1e-6
    assert fixattn.fix_attn_workspace_bytes(p, False) > fixattn.NOALLOC_MAX_WORKSPACE_BYTES
    buf = torch.empty(64, dtype=torch.uint8, device="cuda")     # never touched
    ptrs = [_ptr(buf)] * 9
    s = lib.fix_attn_fwd_noalloc(ctypes.byref(p), *ptrs, None)
    assert s == FIX_ERR_WORKSPACE

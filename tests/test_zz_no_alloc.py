"""fix_attn_fwd_noalloc: the forward for callers that cannot allocate.

Some callers have no device allocator at hand when they call the forward
(host code given only tensors and a stream, or a runtime whose device memory
is fixed up front).  fix_attn_fwd_noalloc serves them from a fixed device
array inside the library.  These tests call it through the C ABI and check
that two calls in a row (different inputs, so nothing stale from the first
call may leak into the second) give exactly the outputs of the ordinary entry
point: both run the same kernels on the same inputs, only the workspace's
address differs.  Problems just under and just over the array's size check
the size limit where it bites.  After every call the array's device status
word is read through fix_attn_noalloc_device_status.  This file is collected
last so that a failure here stops a run only after every other test ran.
"""
import ctypes

import pytest
import torch

import synth

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
                                 _ptr(t["g"]), _ptr(t["w"]), None, _ptr(y), _ptr(o), _ptr(m),
                                 _ptr(r), stream)
    torch.cuda.synchronize()
    del keep
    return s, y, (o, m, r)


def _inputs(seed, seqlens=None, B=2, T=300, Hq=4, Hkv=2, D=64):
    case = synth.make_case(B, T, Hq, Hkv, D, D, seed=seed, seqlens=seqlens)
    t = {k: case[k].cuda().contiguous() for k in ("q", "k", "v", "g", "w")}
    cu = case["cu_seqlens"]
    return t, (cu.cuda() if cu is not None else None), cu


def _same_as_workspace_forward(lib, fixattn, t, cu, cu_host):
    s, y, saved = _noalloc_call(lib, fixattn, t, cu, cu_host)
    assert s == 0, fixattn.status_string(s)
    assert fixattn.fix_attn_noalloc_device_status() == 0
    y_ref, saved_ref = fixattn.fix_attn_fwd(t["q"], t["k"], t["v"], t["g"], t["w"], cu,
                                            cu_host, y_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    for x, xr in zip(saved, saved_ref):
        assert torch.equal(x, xr)


def _problem(fixattn, T, Hq=8, Hkv=4, D=128):
    p = fixattn.Problem()
    p.batch, p.seqlen, p.num_q_heads, p.num_kv_heads = 1, T, Hq, Hkv
    p.head_dim_k = p.head_dim_v = D
    p.eps = 1e-6
    return p


def _largest_fitting_T(fixattn, **kw):
    """Largest T whose forward workspace fits the array (bisection on the
    library's own size function, so it follows the workspace layout)."""
    lo, hi = 1, 1 << 20
    cap = fixattn.NOALLOC_MAX_WORKSPACE_BYTES
    assert fixattn.fix_attn_workspace_bytes(_problem(fixattn, hi, **kw), False) > cap
    while hi - lo > 1:
        mid = (lo + hi) // 2
        if fixattn.fix_attn_workspace_bytes(_problem(fixattn, mid, **kw), False) <= cap:
            lo = mid
        else:
            hi = mid
    return lo


def test_noalloc_forward_matches_workspace_forward_two_calls(cuda_lib):
    from gated_softmax_attention_fp32_b200 import fixattn
    lib = fixattn.load()
    for seed, seqlens in ((11, None), (12, [5, 0, 260, 1, 140])):
        t, cu, cu_host = _inputs(seed, seqlens, B=1 if seqlens else 2)
        _same_as_workspace_forward(lib, fixattn, t, cu, cu_host)


def test_noalloc_at_and_beyond_its_size_limit(cuda_lib):
    """The largest problem that fits the array uses it (nearly) whole and
    still equals the ordinary forward; one token more is rejected with
    FIX_ERR_WORKSPACE before any launch."""
    from gated_softmax_attention_fp32_b200 import fixattn
    lib = fixattn.load()
    T = _largest_fitting_T(fixattn)
    need = fixattn.fix_attn_workspace_bytes(_problem(fixattn, T), False)
    assert need > fixattn.NOALLOC_MAX_WORKSPACE_BYTES - 64 * 1024
    t, cu, cu_host = _inputs(21, None, B=1, T=T, Hq=8, Hkv=4, D=128)
    _same_as_workspace_forward(lib, fixattn, t, cu, cu_host)
    t, cu, cu_host = _inputs(22, None, B=1, T=T + 1, Hq=8, Hkv=4, D=128)
    s, _, _ = _noalloc_call(lib, fixattn, t, cu, cu_host)
    assert s == FIX_ERR_WORKSPACE
    # the rejected call launched nothing: the array still holds a clean status
    assert fixattn.fix_attn_noalloc_device_status() == 0


def test_noalloc_rejects_problem_far_beyond_its_workspace(cuda_lib):
    from gated_softmax_attention_fp32_b200 import fixattn
    lib = fixattn.load()
    p = _problem(fixattn, 1 << 16, Hq=8, Hkv=8)
    assert fixattn.fix_attn_workspace_bytes(p, False) > fixattn.NOALLOC_MAX_WORKSPACE_BYTES
    buf = torch.empty(64, dtype=torch.uint8, device="cuda")     # never touched
    ptrs = [_ptr(buf)] * 10
    s = lib.fix_attn_fwd_noalloc(ctypes.byref(p), *ptrs, None)
    assert s == FIX_ERR_WORKSPACE

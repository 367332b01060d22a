"""Device-side failure detection without a GPU fault or a hang.

Every mbarrier wait in the tensor-core kernels is bounded; one that expires
records FIX_ERR_DEVICE_TIMEOUT in the workspace status word, sets the CTA's
abort flag so that every warp role leaves, waits for its own copies in
flight and releases TMEM.  The test build of the library
(libfixattn_test.so, compiled with -DFIX_TEST_HOOKS) can run the forward
"stalled": its producer warp issues no loads (nothing is ever in flight) and
every wait gives up after 1 ms.  This test makes those waits run out on a
small problem, checks the status word, and checks that the next ordinary call
on the same workspace succeeds and matches the product library bit for bit.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

FIX_OK, FIX_ERR_DEVICE_TIMEOUT = 0, 10


def _test_lib():
    from gated_softmax_attention_fp32_b200 import fixattn
    path = os.path.join(os.path.dirname(fixattn.LIB_PATH), "libfixattn_test.so")
    if not os.path.exists(path):
        pytest.fail(f"test build of the library missing: {path}")
    lib = ctypes.CDLL(path)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.fix_attn_fwd.argtypes = [ctypes.POINTER(fixattn.Problem)] + [vp] * 11 + [sz, vp]
    lib.fix_attn_fwd.restype = ctypes.c_int
    lib.fix_attn_device_status.argtypes = [vp, vp]
    lib.fix_attn_device_status.restype = ctypes.c_int
    lib.fix_attn_workspace_bytes.argtypes = [ctypes.POINTER(fixattn.Problem), ctypes.c_int]
    lib.fix_attn_workspace_bytes.restype = sz
    lib.fix_attn_test_stall_forward.argtypes = [ctypes.c_int]
    lib.fix_attn_test_stall_forward.restype = None
    return lib


def test_forward_wait_expiry_reports_timeout_and_recovers(cuda_lib):
    from gated_softmax_attention_fp32_b200 import fixattn
    lib = _test_lib()
    case = synth.make_case(1, 300, 4, 2, 64, 64, seed=5)
    t = {k: case[k].cuda().contiguous() for k in ("q", "k", "v", "g", "w")}
    p, keep = fixattn.make_problem(t["q"], t["k"], t["v"], None, None, None, case["eps"],
                                   torch.float32)
    ws = torch.empty(lib.fix_attn_workspace_bytes(ctypes.byref(p), 0), device="cuda",
                     dtype=torch.uint8)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    y = torch.full((1, 300, 4, 64), float("nan"), device="cuda")

    def call():
        ptr = lambda x: ctypes.c_void_p(x.data_ptr())
        return lib.fix_attn_fwd(ctypes.byref(p), ptr(t["q"]), ptr(t["k"]), ptr(t["v"]),
                                ptr(t["g"]), ptr(t["w"]), None, ptr(y), None, None, None, ptr(ws),
                                ws.numel(), stream)

    try:
        lib.fix_attn_test_stall_forward(1)
        assert call() == FIX_OK                       # the launch itself is fine
        assert lib.fix_attn_device_status(ptr_of(ws), stream) == FIX_ERR_DEVICE_TIMEOUT
    finally:
        lib.fix_attn_test_stall_forward(0)
    # the context is intact: the same workspace serves an ordinary call
    assert call() == FIX_OK
    assert lib.fix_attn_device_status(ptr_of(ws), stream) == FIX_OK
    ref, _ = fixattn.fix_attn_fwd(t["q"], t["k"], t["v"], t["g"], t["w"], y_dtype=torch.float32,
                                  save=False)
    torch.cuda.synchronize()
    assert torch.equal(y, ref)
    assert np.isfinite(y.cpu().numpy()).all()
    del keep


def ptr_of(x):
    return ctypes.c_void_p(x.data_ptr())

"""The forward's polynomial 2^x against exact powers of two.

Half of the softmax exponentials in the tensor-core forward are evaluated on
the FMA pipe: Cody-Waite reduction to f in [-1/2, 1/2], a degree-3 polynomial
for 2^f, and the integer part added to the exponent field.  Its results feed
16-bit tensor-core operands (and fp32 row sums), so the bound it must meet is
below fp16's half-ulp, 2^-11 ~ 4.9e-4; the fit reaches 7.5e-5.  The test build
of the library exposes the device function on an array of floats.
"""
import ctypes
import os

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

REL_BOUND = 7.6e-5


def _lib():
    from gated_softmax_attention_fp32_b200 import fixattn
    path = os.path.join(os.path.dirname(fixattn.LIB_PATH), "libfixattn_test.so")
    if not os.path.exists(path):
        pytest.fail(f"test build of the library missing: {path}")
    lib = ctypes.CDLL(path)
    for fn in (lib.fix_attn_test_exp2_poly, lib.fix_attn_test_exp2_poly_x2):
        fn.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p]
        fn.restype = ctypes.c_int
    return lib


def _run(lib, x, paired=False):
    xd = torch.from_numpy(x).cuda()
    out = torch.empty_like(xd)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    fn = lib.fix_attn_test_exp2_poly_x2 if paired else lib.fix_attn_test_exp2_poly
    assert fn(ctypes.c_void_p(xd.data_ptr()), ctypes.c_void_p(out.data_ptr()), x.size, stream) == 0
    torch.cuda.synchronize()
    return out.cpu().numpy(), torch.exp2(xd).cpu().numpy()


@pytest.mark.parametrize("paired", [False, True])
def test_exp2_poly_relative_error(cuda_lib, paired):
    lib = _lib()
    # the softmax arguments: <= 0 after the row max, down to where fp16 flushes
    dense = np.linspace(-30.0, 0.0, 3_000_001, dtype=np.float32)
    # every reduced argument pattern near the rounding boundaries of n
    edges = (np.arange(-30, 12, dtype=np.float32)[:, None]
             + np.array([-0.5, -0.4999999, 0.4999999, 0.5, 0.0], dtype=np.float32)).ravel()
    x = np.concatenate([dense, edges.astype(np.float32), np.array([12.0], np.float32)])
    got, cuda_exp2 = _run(lib, x, paired)
    exact = np.exp2(x.astype(np.float64))
    rel = np.abs(got.astype(np.float64) - exact) / exact
    assert rel.max() <= REL_BOUND, float(rel.max())
    # and consistent with the library exp2 well inside fp16 rounding
    rel_cuda = np.abs(got.astype(np.float64) - cuda_exp2) / cuda_exp2
    assert rel_cuda.max() <= REL_BOUND + 2e-7


@pytest.mark.parametrize("paired", [False, True])
def test_exp2_poly_underflow_is_tiny(cuda_lib, paired):
    lib = _lib()
    x = np.array([-126.0, -200.0, -1e30, -np.inf, -127.5], dtype=np.float32)
    got, _ = _run(lib, x, paired)
    # clamped at 2^-125: far below fp16's smallest subnormal, never NaN or negative
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got <= 2.0 ** -124)

"""Python binding of libfixattn.so (include/fix_attn.h): argument marshalling only.

Every step of FiX attention runs in the library's CUDA kernels; this module
allocates the output tensors and the workspace with PyTorch, passes raw device
pointers and the current CUDA stream through ctypes, and turns status codes
into exceptions.  There is no fallback: if the library is missing or the
device is not a B200 (sm_100), calls raise.

Names mirror the C ABI: ``fix_attn_fwd``, ``fix_attn_bwd``,
``fix_attn_workspace_bytes``, ``fix_attn_device_status``; ``fix_attn`` wraps
the pair in a ``torch.autograd.Function`` with the FiX README's argument order
("Quick Start": q, k, v, g, then cu_seqlens / o_norm_weight).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = ["load", "Problem", "fix_attn_fwd", "fix_attn_bwd", "fix_attn_workspace_bytes",
           "fix_attn_decode",
           "fix_attn_device_status", "fix_attn", "training_workspace", "FixStatusError", "LIB_PATH",
           "EXPORTS"]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfixattn.so")
EXPORTS = ("fix_attn_workspace_bytes", "fix_attn_fwd", "fix_attn_bwd", "fix_attn_device_status",
           "fix_attn_kernel_count", "fix_attn_status_string", "fix_attn_fwd_noalloc",
           "fix_attn_noalloc_device_status", "fix_attn_decode_workspace_bytes",
           "fix_attn_decode")
NOALLOC_MAX_WORKSPACE_BYTES = 16 * 1024 * 1024
FIX_FLAG_REUSE_FWD_WORKSPACE = 1
FIX_FLAG_NO_NORM = 2
FIX_FLAG_SCALAR_GATE = 4
STAGES = ("fwd_prefix", "fwd_attn", "bwd_prefix", "bwd_pre", "bwd_dq", "bwd_dkv", "bwd_dg",
          "bwd_finish")

ALGOS = {"auto": 0, "simt": 1, "tc": 2}
_lib = None


class Problem(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("seqlen", ctypes.c_int32),
                ("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim_k", ctypes.c_int32), ("head_dim_v", ctypes.c_int32),
                ("num_seqs", ctypes.c_int32), ("y_dtype", ctypes.c_int32),
                ("algo", ctypes.c_int32), ("flags", ctypes.c_int32),
                ("cu_seqlens", ctypes.c_void_p), ("cu_seqlens_host", ctypes.c_void_p),
                ("scale", ctypes.c_float), ("eps", ctypes.c_float),
                ("events", ctypes.c_void_p)]


class FixStatusError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (code {code})")


def load():
    """Load libfixattn.so (once).  Raises if it is missing: there is no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"FiX CUDA library not built: {LIB_PATH} is missing "
                           "(run python -m gated_softmax_attention_fp32_b200.build)")
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.POINTER(Problem)
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.fix_attn_workspace_bytes.argtypes = [P, ctypes.c_int]
    lib.fix_attn_workspace_bytes.restype = sz
    lib.fix_attn_fwd.argtypes = [P] + [vp] * 11 + [sz, vp]
    lib.fix_attn_fwd.restype = ctypes.c_int
    lib.fix_attn_bwd.argtypes = [P] + [vp] * 17 + [sz, vp]
    lib.fix_attn_bwd.restype = ctypes.c_int
    lib.fix_attn_fwd_noalloc.argtypes = [P] + [vp] * 10 + [vp]
    lib.fix_attn_fwd_noalloc.restype = ctypes.c_int
    lib.fix_attn_device_status.argtypes = [vp, vp]
    lib.fix_attn_device_status.restype = ctypes.c_int
    lib.fix_attn_noalloc_device_status.argtypes = [vp]
    lib.fix_attn_noalloc_device_status.restype = ctypes.c_int
    lib.fix_attn_decode_workspace_bytes.argtypes = [P]
    lib.fix_attn_decode_workspace_bytes.restype = sz
    lib.fix_attn_decode.argtypes = [P] + [vp] * 9 + [sz, vp]
    lib.fix_attn_decode.restype = ctypes.c_int
    lib.fix_attn_kernel_count.argtypes = [P, ctypes.c_int]
    lib.fix_attn_kernel_count.restype = ctypes.c_int
    lib.fix_attn_status_string.argtypes = [ctypes.c_int]
    lib.fix_attn_status_string.restype = ctypes.c_char_p
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load().fix_attn_status_string(int(code)).decode()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def make_problem(q, k, v, cu_seqlens=None, cu_seqlens_host=None, scale=None, eps=1e-6,
                 y_dtype=torch.bfloat16, algo="auto", events=None, o_norm=True,
                 scalar_gate=False):
    """Build the C problem descriptor from [B,T,H,D] tensors.  Returns
    (Problem, keepalive) where keepalive holds the host cu_seqlens tensor and
    the event-handle array.  ``events``: optional list of 2*len(STAGES)
    ``torch.cuda.Event(enable_timing=True)`` recorded around each stage.
    ``o_norm=False`` sets FIX_FLAG_NO_NORM, ``scalar_gate`` (g of shape
    [B,T,Hkv]) FIX_FLAG_SCALAR_GATE."""
    B, T, Hq, Dk = q.shape
    Hkv, Dv = v.shape[2], v.shape[3]
    p = Problem()
    p.batch, p.seqlen, p.num_q_heads, p.num_kv_heads = B, T, Hq, Hkv
    p.head_dim_k, p.head_dim_v = Dk, Dv
    p.y_dtype = 1 if y_dtype == torch.float32 else 0
    p.algo = ALGOS[algo]
    p.flags = (0 if o_norm else FIX_FLAG_NO_NORM) | (FIX_FLAG_SCALAR_GATE if scalar_gate else 0)
    p.scale = float(scale) if scale is not None else 0.0
    p.eps = float(eps)
    keep = None
    if cu_seqlens is not None:
        if cu_seqlens_host is None:
            cu_seqlens_host = cu_seqlens.detach().to("cpu")
        keep = cu_seqlens_host.to(torch.int64).contiguous()
        p.num_seqs = keep.numel() - 1
        p.cu_seqlens = cu_seqlens.data_ptr()
        p.cu_seqlens_host = keep.data_ptr()
    else:
        p.num_seqs = 0
    if events is not None:
        assert len(events) == 2 * len(STAGES)
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        p.events = ctypes.cast(arr, ctypes.c_void_p)
        keep = (keep, arr)
    return p, keep


def fix_attn_workspace_bytes(problem: Problem, backward: bool) -> int:
    return int(load().fix_attn_workspace_bytes(ctypes.byref(problem), int(bool(backward))))


def fix_attn_kernel_count(problem: Problem, backward: bool) -> int:
    return int(load().fix_attn_kernel_count(ctypes.byref(problem), int(bool(backward))))


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def fix_attn_fwd(q, k, v, g, o_norm_weight, cu_seqlens=None, cu_seqlens_host=None, scale=None,
                 eps=1e-6, y_dtype=torch.bfloat16, save=True, algo="auto", workspace=None,
                 out=None, stream=None, events=None, o_gate=None, o_norm=True):
    """Forward.  Returns (y, saved) with saved = (o, m, rstd) or None.  g of
    shape [B,T,Hkv] is a scalar gate; ``o_gate`` [B,T,Hq,Dv] bf16 gates the
    output with swish; ``o_norm=False`` drops the RMSNorm (o_norm_weight may
    then be None)."""
    lib = load()
    p, keep = make_problem(q, k, v, cu_seqlens, cu_seqlens_host, scale, eps, y_dtype, algo,
                           events, o_norm, g.dim() == 3)
    B, T, Hq, _ = q.shape
    Dv = v.shape[3]
    dev = q.device
    y = out if out is not None else torch.empty(B, T, Hq, Dv, device=dev, dtype=y_dtype)
    saved = None
    if save:
        saved = (torch.empty(B, T, Hq, Dv, device=dev, dtype=torch.float32),
                 torch.empty(B, T, Hq, device=dev, dtype=torch.float32),
                 torch.empty(B, T, Hq, device=dev, dtype=torch.float32))
    nbytes = fix_attn_workspace_bytes(p, False)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), device=dev, dtype=torch.uint8)
    s = lib.fix_attn_fwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o_norm_weight),
                         _ptr(o_gate), _ptr(y),
                         *(map(_ptr, saved) if saved else (None, None, None)),
                         _ptr(workspace), workspace.numel(), _stream(stream))
    if s != 0:
        raise FixStatusError(s, "fix_attn_fwd")
    del keep
    return y, saved


def fix_attn_fwd_noalloc(q, k, v, g, o_norm_weight, y, saved, cu_seqlens=None,
                         cu_seqlens_host=None, scale=None, eps=1e-6, algo="auto", stream=None,
                         o_gate=None, o_norm=True):
    """Forward into caller-provided ``y`` and ``saved`` = (o, m, rstd) or None,
    with the library's own fixed device workspace (no allocation by anyone)."""
    lib = load()
    p, keep = make_problem(q, k, v, cu_seqlens, cu_seqlens_host, scale, eps, y.dtype, algo,
                           None, o_norm, g.dim() == 3)
    s = lib.fix_attn_fwd_noalloc(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                 _ptr(o_norm_weight), _ptr(o_gate), _ptr(y),
                                 *(map(_ptr, saved) if saved else (None, None, None)),
                                 _stream(stream))
    if s != 0:
        raise FixStatusError(s, "fix_attn_fwd_noalloc")
    del keep
    return y, saved


def fix_attn_bwd(q, k, v, g, o_norm_weight, dy, saved, cu_seqlens=None, cu_seqlens_host=None,
                 scale=None, eps=1e-6, algo="auto", workspace=None, stream=None, events=None,
                 out=None, reuse_forward_workspace=False, o_gate=None, o_norm=True):
    """Backward of sum(dy * y).  Returns dq, dk, dv, dg, dw, d_o_gate (the last
    None without an output gate; dw None without the norm and no ``out``)
    (``out`` may supply those six tensors).  ``reuse_forward_workspace``:
    ``workspace`` is the one the matching training forward used (sized for the
    backward, see ``training_workspace``) and has not been written since; the
    backward then reuses the forward's gate prefix results
    (FIX_FLAG_REUSE_FWD_WORKSPACE)."""
    lib = load()
    p, keep = make_problem(q, k, v, cu_seqlens, cu_seqlens_host, scale, eps, torch.bfloat16, algo,
                           events, o_norm, g.dim() == 3)
    if reuse_forward_workspace:
        if workspace is None:
            raise ValueError("reuse_forward_workspace needs the forward's workspace")
        p.flags |= FIX_FLAG_REUSE_FWD_WORKSPACE
    if out is not None:
        dq, dk, dv, dg, dw = out[:5]
        dz = out[5] if len(out) > 5 else None
    else:
        dq = torch.empty_like(q)
        dk = torch.empty_like(k)
        dv = torch.empty_like(v)
        dg = torch.empty_like(g)
        dw = torch.empty_like(o_norm_weight) if o_norm_weight is not None else None
        dz = None
    if o_gate is not None and dz is None:
        dz = torch.empty_like(o_gate)
    nbytes = fix_attn_workspace_bytes(p, True)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), device=q.device, dtype=torch.uint8)
    o_s, m_s, r_s = saved
    s = lib.fix_attn_bwd(ctypes.byref(p), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o_norm_weight),
                         _ptr(o_gate), _ptr(dy), _ptr(o_s), _ptr(m_s), _ptr(r_s), _ptr(dq),
                         _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dw), _ptr(dz), _ptr(workspace),
                         workspace.numel(), _stream(stream))
    if s != 0:
        raise FixStatusError(s, "fix_attn_bwd")
    del keep
    return dq, dk, dv, dg, dw, dz


def training_workspace(q, k, v, cu_seqlens=None, cu_seqlens_host=None, algo="auto", g=None,
                       o_norm=True):
    """A workspace sized for the backward, to pass to a training forward and
    then to its backward with ``reuse_forward_workspace=True``."""
    p, keep = make_problem(q, k, v, cu_seqlens, cu_seqlens_host, None, 1e-6, torch.bfloat16, algo,
                           None, o_norm, g is not None and g.dim() == 3)
    n = fix_attn_workspace_bytes(p, True)
    del keep
    return torch.empty(max(n, 1), device=q.device, dtype=torch.uint8)


def fix_attn_decode(q, k_cache, v_cache, g_cache, seqlens, o_norm_weight=None, scale=None,
                    eps=1e-6, y_dtype=torch.bfloat16, o_gate=None, o_norm=True, workspace=None,
                    out=None, stream=None):
    """One new query per sequence against its cache.  q [B,Hq,Dk];
    k_cache [B,Tmax,Hkv,Dk], v_cache [B,Tmax,Hkv,Dv] bf16; g_cache
    [B,Tmax,Hkv,Dv] (or [B,Tmax,Hkv]) f32; seqlens int32 [B] on the device
    (tokens per cache, the new one included).  Returns y [B,Hq,Dv]."""
    lib = load()
    B, Hq, Dk = q.shape
    Tmax, Hkv, Dv = v_cache.shape[1], v_cache.shape[2], v_cache.shape[3]
    p = Problem()
    p.batch, p.seqlen, p.num_q_heads, p.num_kv_heads = B, Tmax, Hq, Hkv
    p.head_dim_k, p.head_dim_v = Dk, Dv
    p.y_dtype = 1 if y_dtype == torch.float32 else 0
    p.flags = (0 if o_norm else FIX_FLAG_NO_NORM) | (FIX_FLAG_SCALAR_GATE if g_cache.dim() == 3 else 0)
    p.scale = float(scale) if scale is not None else 0.0
    p.eps = float(eps)
    y = out if out is not None else torch.empty(B, Hq, Dv, device=q.device, dtype=y_dtype)
    nbytes = int(lib.fix_attn_decode_workspace_bytes(ctypes.byref(p)))
    if workspace is None:
        workspace = torch.empty(max(nbytes, 1), device=q.device, dtype=torch.uint8)
    s = lib.fix_attn_decode(ctypes.byref(p), _ptr(seqlens), _ptr(q), _ptr(k_cache), _ptr(v_cache),
                            _ptr(g_cache), _ptr(o_norm_weight), _ptr(o_gate), _ptr(y),
                            _ptr(workspace), workspace.numel(), _stream(stream))
    if s != 0:
        raise FixStatusError(s, "fix_attn_decode")
    return y


def fix_attn_device_status(workspace, stream=None) -> int:
    return int(load().fix_attn_device_status(_ptr(workspace), _stream(stream)))


def fix_attn_noalloc_device_status(stream=None) -> int:
    """Device status word of the last fix_attn_fwd_noalloc call on the current
    device (synchronises the stream)."""
    return int(load().fix_attn_noalloc_device_status(_stream(stream)))


def _check(ws, where):
    s = fix_attn_device_status(ws)
    if s != 0:
        raise FixStatusError(s, where)


class _FixAttn(torch.autograd.Function):
    @staticmethod
    def forward(ctx, q, k, v, g, w, z, cu_seqlens, cu_host, scale, eps, algo, o_norm, check):
        ws = training_workspace(q, k, v, cu_seqlens, cu_host, algo, g, o_norm)
        y, saved = fix_attn_fwd(q, k, v, g, w, cu_seqlens, cu_host, scale, eps, save=True,
                                algo=algo, workspace=ws, o_gate=z, o_norm=o_norm)
        if check:
            _check(ws, "fix_attn forward (device status)")
        ctx.save_for_backward(q, k, v, g, w, z, *saved)
        ctx.cfg = (cu_seqlens, cu_host, scale, eps, algo, o_norm, check)
        ctx.ws = ws
        return y

    @staticmethod
    def backward(ctx, dy):
        q, k, v, g, w, z, o_s, m_s, r_s = ctx.saved_tensors
        cu, cu_host, scale, eps, algo, o_norm, check = ctx.cfg
        dq, dk, dv, dg, dw, dz = fix_attn_bwd(q, k, v, g, w, dy.to(torch.bfloat16).contiguous(),
                                              (o_s, m_s, r_s), cu, cu_host, scale, eps, algo,
                                              workspace=ctx.ws, reuse_forward_workspace=True,
                                              o_gate=z, o_norm=o_norm)
        if check:
            _check(ctx.ws, "fix_attn backward (device status)")
        ctx.ws = None
        return dq, dk, dv, dg, dw, dz, None, None, None, None, None, None, None


def fix_attn(q, k, v, g, o_norm_weight=None, cu_seqlens=None, cu_seqlens_host=None, scale=None,
             eps=1e-6, algo="auto", o_gate=None, o_norm=True, check_status=True):
    """FiX attention, differentiable, with the FiX README's arguments ("Quick
    Start"): y = RMSNorm(FiX attention(q, k, v, g)) * o_norm_weight
    [* swish(o_gate)]; with ``o_norm=False`` the output is the attention
    average o_t / l_t [* swish(o_gate)].  g [B,T,Hkv,Dv] (element-wise gate)
    or [B,T,Hkv] (scalar gate).  ``check_status`` reads the device status
    word after the forward and after the backward (each read synchronises
    the stream) and raises FixStatusError if a bounded device wait expired;
    pass False to keep the calls asynchronous."""
    if o_norm and o_norm_weight is None:
        raise ValueError("o_norm=True needs o_norm_weight")
    return _FixAttn.apply(q, k, v, g, o_norm_weight, o_gate, cu_seqlens, cu_seqlens_host, scale,
                          eps, algo, o_norm, check_status)

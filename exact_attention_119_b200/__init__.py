"""exact_attention_119_b200: exact attention on B200 (sm_100a) behind a C ABI.

This module is argument marshalling only: it checks torch tensors, hands raw
device pointers, sizes and the current CUDA stream to ``libfa.so`` (built
in-tree by ``exact_attention_119_b200.build``) and returns the tensors it
allocated. Every step of the computation runs in the library's kernels; there
is no CPU or PyTorch fallback. If the library is missing or cannot load, the
first call raises.

Interface, after ``flash_attn_func`` as described by the lab write-up
"从Attention矩阵到显存读写：FlashAttention真正解决的痛点" (§4.2): q, k, v are
[batch, seqlen, heads, head_dim] fp16/bf16 tensors (fp32 is an error),
``softmax_scale=None`` means 1/sqrt(head_dim), ``causal`` masks keys after the
query.
"""

from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "forward", "backward", "flash_attn_func", "bwd_workspace_size", "check_device_status",
    "status_string", "library", "FAError", "LIB_PATH",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")

FA_OK = 0
FA_FP16 = 0
FA_BF16 = 1

_lib = None


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} ({status})")


def library() -> ctypes.CDLL:
    """The loaded libfa.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libfa.so not built at {LIB_PATH}; run python -m exact_attention_119_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
        lib.fa_fwd.restype = i
        lib.fa_bwd_workspace_size.argtypes = [i, i, i, i, i]
        lib.fa_bwd_workspace_size.restype = sz
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, i, vp]
        lib.fa_bwd.restype = i
        lib.fa_check_device_status.argtypes = [vp]
        lib.fa_check_device_status.restype = i
        lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
        lib.fa_bwd_noalloc.restype = i
        lib.fa_selftest_bounded_wait.argtypes = [i, i, vp]
        lib.fa_selftest_bounded_wait.restype = i
        lib.fa_status_string.argtypes = [i]
        lib.fa_status_string.restype = ctypes.c_char_p
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().fa_status_string(int(status)).decode()


def _dtype_code(t):
    import torch
    if t.dtype == torch.float16:
        return FA_FP16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    raise TypeError(f"attention inputs must be float16 or bfloat16, got {t.dtype}")


def _check_bnhd(name, t, like=None):
    if t.dim() != 4:
        raise ValueError(f"{name} must be [batch, seqlen, heads, head_dim], got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if like is not None and (t.shape != like.shape or t.dtype != like.dtype or t.device != like.device):
        raise ValueError(f"{name} must match q in shape, dtype and device")


def _stream_ptr(stream):
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _scale(softmax_scale, d):
    return 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)


def forward(q, k, v, softmax_scale=None, causal=False, out=None, lse=None, stream=None):
    """O = softmax(scale Q K^T [+causal]) V and the row LSE [B, H, N] fp32."""
    import torch
    code = _dtype_code(q)
    _check_bnhd("q", q)
    _check_bnhd("k", k, q)
    _check_bnhd("v", v, q)
    B, N, H, d = q.shape
    if out is None:
        out = torch.empty_like(q)
    else:
        _check_bnhd("out", out, q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    st = library().fa_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), lse.data_ptr(),
                          B, N, H, d, _scale(softmax_scale, d), int(bool(causal)), code, _stream_ptr(stream))
    if st != FA_OK:
        raise FAError(st, "fa_fwd")
    return out, lse


def bwd_workspace_size(B, N, H, d, causal=False) -> int:
    return int(library().fa_bwd_workspace_size(B, N, H, d, int(bool(causal))))


def backward(q, k, v, o, dout, lse, softmax_scale=None, causal=False, dq=None, dk=None, dv=None,
             workspace=None, stream=None):
    """Gradients (dQ, dK, dV) given dout = dL/dO and the forward's O and LSE."""
    import torch
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_bnhd(name, t, q)
    B, N, H, d = q.shape
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [B, H, N] float32 tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    need = bwd_workspace_size(B, N, H, d, causal)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    st = library().fa_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(), lse.data_ptr(),
                          dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(), workspace.numel(),
                          B, N, H, d, _scale(softmax_scale, d), int(bool(causal)), code, _stream_ptr(stream))
    if st != FA_OK:
        raise FAError(st, "fa_bwd")
    return dq, dk, dv


def backward_noalloc(q, k, v, o, dout, lse, softmax_scale=None, causal=False, dq=None, dk=None, dv=None,
                     stream=None):
    """backward() through fa_bwd_noalloc: the library's built-in scratch instead
    of a workspace, for callers that cannot allocate device memory (the output
    tensors are still the caller's). Calls that overlap on the GPU race on the
    shared scratch; shapes needing more than noalloc_max_workspace() bytes of
    scratch raise FAError (FA_ERR_WORKSPACE)."""
    import torch
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_bnhd(name, t, q)
    B, N, H, d = q.shape
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [B, H, N] float32 tensor")
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    st = library().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                  lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, N, H, d,
                                  _scale(softmax_scale, d), int(bool(causal)), code, _stream_ptr(stream))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_noalloc")
    return dq, dk, dv


# Size of the built-in scratch behind fa_bwd_noalloc (stated in include/fa.h).
NOALLOC_MAX_WORKSPACE = 32 << 20


def noalloc_max_workspace() -> int:
    return NOALLOC_MAX_WORKSPACE


def check_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return int(library().fa_check_device_status(_stream_ptr(stream)))


def selftest_bounded_wait(which: int, limit_ms: int = 50, stream=None) -> None:
    """Launch the failure-detection self-test kernel (see include/fa.h)."""
    st = library().fa_selftest_bounded_wait(int(which), int(limit_ms), _stream_ptr(stream))
    if st != FA_OK:
        raise FAError(st, "fa_selftest_bounded_wait")


def _autograd_function():
    import torch

    class _FlashAttention(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, softmax_scale, causal):
            o, lse = forward(q, k, v, softmax_scale, causal)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.softmax_scale = softmax_scale
            ctx.causal = causal
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse = ctx.saved_tensors
            dq, dk, dv = backward(q, k, v, o, do.contiguous(), lse, ctx.softmax_scale, ctx.causal)
            return dq, dk, dv, None, None

    return _FlashAttention


_fn = None


def flash_attn_func(q, k, v, softmax_scale=None, causal=False):
    """Differentiable exact attention on [B, N, H, d] fp16/bf16 CUDA tensors."""
    global _fn
    if _fn is None:
        _fn = _autograd_function()
    return _fn.apply(q, k, v, softmax_scale, causal)

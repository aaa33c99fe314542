"""exact_attention_119_b200: exact attention on B200 (sm_100a) behind a C ABI.

This module is argument marshalling only: it checks torch tensors, hands raw
device pointers, strides, sizes and the current CUDA stream to ``libfa.so``
(built in-tree by ``exact_attention_119_b200.build``) and returns the tensors
it allocated. Every step of the computation runs in the library's kernels;
there is no CPU or PyTorch fallback. If the library is missing or cannot load,
the first call raises.

Interface, after ``flash_attn_func`` as described by the lab write-up
"从Attention矩阵到显存读写：FlashAttention真正解决的痛点" (§4.2): q, k, v are
[batch, seqlen, heads, head_dim] fp16/bf16 tensors (fp32 is an error),
``softmax_scale=None`` means 1/sqrt(head_dim), ``causal`` masks keys after the
query. Tensors may be strided views (head_dim contiguous, other strides
multiples of 8 elements): ``flash_attn_qkvpacked_func`` takes the packed
[B, N, 3, H, d] tensor of "使用FlashAttention优化PyTorch模型注意力计算", and
``flash_attn_varlen_func`` takes sequences packed without padding with their
row offsets (the write-up's §4.2, third pitfall). Head sizes are multiples of
8 up to 128.
"""

from __future__ import annotations

import ctypes
import math
import os

__all__ = [
    "forward", "backward", "backward_noalloc", "flash_attn_func", "flash_attn_qkvpacked_func",
    "flash_attn_varlen_func", "varlen_forward", "varlen_backward", "bwd_workspace_size",
    "check_device_status", "status_string", "last_error_detail", "library", "FAError", "LIB_PATH",
    "profile_bwd_events", "check_same_device", "selftest_bounded_wait", "noalloc_max_workspace",
    "decode", "flash_attn_with_kvcache", "decode_workspace_size",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa.so")

FA_OK = 0
FA_FP16 = 0
FA_BF16 = 1

_lib = None


class FaStrides(ctypes.Structure):
    """fa_strides of include/fa.h: element strides of a [B, N, H, d] view."""
    _fields_ = [("batch", ctypes.c_longlong), ("row", ctypes.c_longlong), ("head", ctypes.c_longlong)]


class FaDesc(ctypes.Structure):
    """fa_desc of include/fa.h."""
    _fields_ = [("B", ctypes.c_int), ("N", ctypes.c_int), ("H", ctypes.c_int), ("d", ctypes.c_int),
                ("softmax_scale", ctypes.c_float), ("causal", ctypes.c_int), ("dtype", ctypes.c_int),
                ("stride_q", FaStrides), ("stride_k", FaStrides), ("stride_v", FaStrides),
                ("stride_o", FaStrides), ("stride_do", FaStrides), ("stride_dq", FaStrides),
                ("stride_dk", FaStrides), ("stride_dv", FaStrides),
                ("cu_seqlens", ctypes.c_void_p), ("total", ctypes.c_int),
                ("dropout_p", ctypes.c_float), ("seed", ctypes.c_ulonglong), ("offset", ctypes.c_uint)]


class FAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.detail = last_error_detail()
        extra = f": {self.detail}" if self.detail else ""
        super().__init__(f"{where}: {status_string(status)} ({status}){extra}")


def library() -> ctypes.CDLL:
    """The loaded libfa.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libfa.so not built at {LIB_PATH}; run python -m exact_attention_119_b200.build")
        lib = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        dp = ctypes.POINTER(FaDesc)
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
        lib.fa_fwd.restype = i
        lib.fa_fwd_ex.argtypes = [dp, vp, vp, vp, vp, vp, vp]
        lib.fa_fwd_ex.restype = i
        lib.fa_bwd_workspace_size.argtypes = [i, i, i, i, i]
        lib.fa_bwd_workspace_size.restype = sz
        lib.fa_bwd_ex_workspace_size.argtypes = [dp]
        lib.fa_bwd_ex_workspace_size.restype = sz
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, f, i, i, vp]
        lib.fa_bwd.restype = i
        lib.fa_bwd_ex.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
        lib.fa_bwd_ex.restype = i
        lib.fa_check_device_status.argtypes = [vp]
        lib.fa_check_device_status.restype = i
        lib.fa_bwd_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
        lib.fa_bwd_noalloc.restype = i
        lib.fa_selftest_bounded_wait.argtypes = [i, i, vp]
        lib.fa_selftest_bounded_wait.restype = i
        lib.fa_status_string.argtypes = [i]
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_last_error_detail.argtypes = []
        lib.fa_last_error_detail.restype = ctypes.c_char_p
        lib.fa_profile_bwd_events.argtypes = [vp, vp]
        lib.fa_profile_bwd_events.restype = i
        lib.fa_decode_workspace_size.argtypes = [i, i, i, i, i]
        lib.fa_decode_workspace_size.restype = sz
        lib.fa_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, sz, i, i, i, i, i, f, i, i, vp]
        lib.fa_decode.restype = i
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return library().fa_status_string(int(status)).decode()


def last_error_detail() -> str:
    """What the last failing library call of this thread ran into ('' if none)."""
    return library().fa_last_error_detail().decode()


def _dtype_code(t):
    import torch
    if t.dtype == torch.float16:
        return FA_FP16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    raise TypeError(f"attention inputs must be float16 or bfloat16, got {t.dtype}")


def _check_view(name, t, like=None, dims=4):
    what = "[batch, seqlen, heads, head_dim]" if dims == 4 else "[total, heads, head_dim]"
    if t.dim() != dims:
        raise ValueError(f"{name} must be {what}, got shape {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.stride(-1) != 1:
        raise ValueError(f"{name} must have a contiguous head_dim axis")
    if like is not None and (t.shape != like.shape or t.dtype != like.dtype or t.device != like.device):
        raise ValueError(f"{name} must match q in shape, dtype and device")


def _strides(t):
    """fa_strides of a [B, N, H, d] or [total, H, d] view. The stride of an
    axis of size 1 is never used; it is given its dense value, so views such
    as x[:, :, None, :] pass the library's stride checks."""
    shape, st = list(t.shape), list(t.stride())
    if t.dim() == 3:
        shape, st = [1] + shape, [0] + st
    dense = [shape[1] * shape[2] * shape[3], shape[2] * shape[3], shape[3]]
    b, n, h = (dense[i] if shape[i] == 1 else st[i] for i in range(3))
    return FaStrides(0 if t.dim() == 3 else b, n, h)


def check_same_device(device, **named):
    """Every named tensor or stream must live on ``device`` (the device of q)."""
    for name, t in named.items():
        if t is not None and t.device != device:
            raise ValueError(f"{name} is on {t.device}, but q is on {device}")


def _stream_ptr(stream, device=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _scale(softmax_scale, d):
    return 1.0 / math.sqrt(d) if softmax_scale is None else float(softmax_scale)


def _desc(ref, softmax_scale, causal, cu_seqlens=None, max_seqlen=None, dropout=None, **tensors):
    """fa_desc of one call; `ref` gives shape and dtype, `tensors` the strides
    (keyword names q, k, v, o, do, dq, dk, dv)."""
    if cu_seqlens is None:
        B, N, H, d = ref.shape
        total = 0
    else:
        total, H, d = ref.shape
        B, N = cu_seqlens.numel() - 1, int(max_seqlen)
    x = FaDesc()
    x.B, x.N, x.H, x.d = B, N, H, d
    x.softmax_scale = _scale(softmax_scale, d)
    x.causal = int(bool(causal))
    x.dtype = _dtype_code(ref)
    x.cu_seqlens = None if cu_seqlens is None else cu_seqlens.data_ptr()
    x.total = total
    if dropout is not None:
        x.dropout_p, x.seed, x.offset = float(dropout[0]), int(dropout[1]), int(dropout[2])
    for name, t in tensors.items():
        setattr(x, "stride_" + name, _strides(t))
    return x


def _run_fwd(desc, q, k, v, out, lse, stream):
    import torch
    check_same_device(q.device, k=k, v=v, out=out, lse=lse, stream=stream)
    with torch.cuda.device(q.device):
        st = library().fa_fwd_ex(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                 lse.data_ptr(), _stream_ptr(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_fwd_ex")


def _dropout(dropout_p, seed, offset):
    if not dropout_p:
        return None
    if not 0.0 <= dropout_p < 1.0:
        raise ValueError("dropout_p must be in [0, 1)")
    if seed is None:
        raise ValueError("dropout needs a seed (the backward regenerates the mask from it)")
    return (dropout_p, seed, offset)


def forward(q, k, v, softmax_scale=None, causal=False, out=None, lse=None, stream=None, dropout_p=0.0, seed=None,
            offset=0):
    """O = softmax(scale Q K^T [+causal]) V and the row LSE [B, H, N] fp32.
    With dropout_p > 0, O = (P o Z) V with Z = keep / (1 - dropout_p), the
    mask drawn from (seed, offset) as include/fa.h states."""
    import torch
    _dtype_code(q)
    _check_view("q", q)
    _check_view("k", k, q)
    _check_view("v", v, q)
    B, N, H, d = q.shape
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    else:
        _check_view("out", out, q)
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    elif lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [B, H, N] float32 tensor")
    _run_fwd(_desc(q, softmax_scale, causal, dropout=_dropout(dropout_p, seed, offset), q=q, k=k, v=v, o=out),
             q, k, v, out, lse, stream)
    return out, lse


def bwd_workspace_size(B, N, H, d, causal=False) -> int:
    return int(library().fa_bwd_workspace_size(B, N, H, d, int(bool(causal))))


def _grad_outputs(q, dq, dk, dv, dims=4):
    import torch
    out = []
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        if t is None:
            t = torch.empty_like(q, memory_format=torch.contiguous_format)
        else:
            _check_view(name, t, q, dims)
        out.append(t)
    return out


def _run_bwd(desc, q, k, v, o, dout, lse, dq, dk, dv, workspace, stream):
    import torch
    need = int(library().fa_bwd_ex_workspace_size(ctypes.byref(desc)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    check_same_device(q.device, k=k, v=v, o=o, dout=dout, lse=lse, dq=dq, dk=dk, dv=dv, workspace=workspace,
                      stream=stream)
    with torch.cuda.device(q.device):
        st = library().fa_bwd_ex(ctypes.byref(desc), q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                 dout.data_ptr(), lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(),
                                 workspace.data_ptr(), workspace.numel(), _stream_ptr(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_ex")


def backward(q, k, v, o, dout, lse, softmax_scale=None, causal=False, dq=None, dk=None, dv=None,
             workspace=None, stream=None, dropout_p=0.0, seed=None, offset=0):
    """Gradients (dQ, dK, dV) given dout = dL/dO and the forward's O and LSE
    (with the forward's dropout_p, seed and offset, if any)."""
    import torch
    _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_view(name, t, q)
    B, N, H, d = q.shape
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [B, H, N] float32 tensor")
    dq, dk, dv = _grad_outputs(q, dq, dk, dv)
    desc = _desc(q, softmax_scale, causal, dropout=_dropout(dropout_p, seed, offset), q=q, k=k, v=v, o=o, do=dout,
                 dq=dq, dk=dk, dv=dv)
    _run_bwd(desc, q, k, v, o, dout, lse, dq, dk, dv, workspace, stream)
    return dq, dk, dv


def backward_noalloc(q, k, v, o, dout, lse, softmax_scale=None, causal=False, dq=None, dk=None, dv=None,
                     stream=None):
    """backward() through fa_bwd_noalloc: the library's built-in scratch instead
    of a workspace, for callers that cannot allocate device memory (the output
    tensors are still the caller's). Dense [B, N, H, d] tensors only. Calls
    that overlap on the GPU race on the shared scratch; shapes needing more
    than noalloc_max_workspace() bytes of scratch raise FAError
    (FA_ERR_WORKSPACE)."""
    import torch
    code = _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_view(name, t, q)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    B, N, H, d = q.shape
    if lse.shape != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [B, H, N] float32 tensor")
    dq, dk, dv = _grad_outputs(q, dq, dk, dv)
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    check_same_device(q.device, lse=lse, stream=stream)
    with torch.cuda.device(q.device):
        st = library().fa_bwd_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), dout.data_ptr(),
                                      lse.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), B, N, H, d,
                                      _scale(softmax_scale, d), int(bool(causal)), code,
                                      _stream_ptr(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_bwd_noalloc")
    return dq, dk, dv


# Size of the built-in scratch behind fa_bwd_noalloc (stated in include/fa.h).
NOALLOC_MAX_WORKSPACE = 32 << 20


def noalloc_max_workspace() -> int:
    return NOALLOC_MAX_WORKSPACE


# ------------------------------------------------------------ variable length

def _check_cu(cu_seqlens, q):
    import torch
    if cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 2:
        raise ValueError("cu_seqlens must be a 1-D int32 tensor of B + 1 row offsets")
    if not cu_seqlens.is_contiguous():
        raise ValueError("cu_seqlens must be contiguous")
    check_same_device(q.device, cu_seqlens=cu_seqlens)


def varlen_forward(q, k, v, cu_seqlens, max_seqlen, softmax_scale=None, causal=False, out=None, lse=None,
                   stream=None, dropout_p=0.0, seed=None, offset=0):
    """Variable-length batch packed without padding: q, k, v are [total, H, d];
    sequence b owns rows cu_seqlens[b] .. cu_seqlens[b+1]-1 (int32 on the
    device) and attends only to itself; max_seqlen bounds every length.
    Returns O [total, H, d] and LSE [H, total] fp32."""
    import torch
    _dtype_code(q)
    _check_view("q", q, dims=3)
    _check_view("k", k, q, dims=3)
    _check_view("v", v, q, dims=3)
    _check_cu(cu_seqlens, q)
    total, H, d = q.shape
    if out is None:
        out = torch.empty_like(q, memory_format=torch.contiguous_format)
    else:
        _check_view("out", out, q, dims=3)
    if lse is None:
        lse = torch.empty((H, total), dtype=torch.float32, device=q.device)
    elif lse.shape != (H, total) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [H, total] float32 tensor")
    desc = _desc(q, softmax_scale, causal, cu_seqlens, max_seqlen, _dropout(dropout_p, seed, offset), q=q, k=k,
                 v=v, o=out)
    _run_fwd(desc, q, k, v, out, lse, stream)
    return out, lse


def varlen_backward(q, k, v, o, dout, lse, cu_seqlens, max_seqlen, softmax_scale=None, causal=False, dq=None,
                    dk=None, dv=None, workspace=None, stream=None, dropout_p=0.0, seed=None, offset=0):
    """Gradients of varlen_forward: dQ, dK, dV [total, H, d]."""
    import torch
    _dtype_code(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _check_view(name, t, q, dims=3)
    _check_cu(cu_seqlens, q)
    total, H, d = q.shape
    if lse.shape != (H, total) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous [H, total] float32 tensor")
    dq, dk, dv = _grad_outputs(q, dq, dk, dv, dims=3)
    desc = _desc(q, softmax_scale, causal, cu_seqlens, max_seqlen, _dropout(dropout_p, seed, offset), q=q, k=k,
                 v=v, o=o, do=dout, dq=dq, dk=dk, dv=dv)
    _run_bwd(desc, q, k, v, o, dout, lse, dq, dk, dv, workspace, stream)
    return dq, dk, dv


# ------------------------------------------------------------ KV-cache decode

def decode_workspace_size(B, Nq, H, d, Nmax) -> int:
    return int(library().fa_decode_workspace_size(B, Nq, H, d, Nmax))


def decode(q, k_cache, v_cache, cache_seqlens, softmax_scale=None, causal=False, out=None, lse=None,
           workspace=None, stream=None):
    """Attention of the Nq newest positions q [B, Nq, H, d] (Nq <= 8) against
    a key/value cache [B, Nmax, H, d] holding cache_seqlens[b] (int32 on the
    device) valid rows per sequence. Returns O [B, Nq, H, d] and LSE
    [B, H, Nq] fp32."""
    import torch
    code = _dtype_code(q)
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_view(name, t)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    B, Nq, H, d = q.shape
    Nmax = k_cache.shape[1]
    if k_cache.shape != (B, Nmax, H, d) or v_cache.shape != k_cache.shape:
        raise ValueError("k_cache and v_cache must be [B, Nmax, H, d] with q's B, H and d")
    if k_cache.dtype != q.dtype or v_cache.dtype != q.dtype:
        raise ValueError("the caches must have q's dtype")
    if cache_seqlens.dtype != torch.int32 or cache_seqlens.shape != (B,) or not cache_seqlens.is_contiguous():
        raise ValueError("cache_seqlens must be a contiguous int32 tensor of B lengths")
    if out is None:
        out = torch.empty_like(q)
    elif out.shape != q.shape or out.dtype != q.dtype or not out.is_contiguous():
        raise ValueError("out must be a contiguous tensor like q")
    if lse is None:
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    need = decode_workspace_size(B, Nq, H, d, Nmax)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    check_same_device(q.device, k_cache=k_cache, v_cache=v_cache, cache_seqlens=cache_seqlens, out=out, lse=lse,
                      workspace=workspace, stream=stream)
    with torch.cuda.device(q.device):
        st = library().fa_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), cache_seqlens.data_ptr(),
                                 out.data_ptr(), lse.data_ptr(), workspace.data_ptr(), workspace.numel(), B, Nq, H,
                                 d, Nmax, _scale(softmax_scale, d), int(bool(causal)), code,
                                 _stream_ptr(stream, q.device))
    if st != FA_OK:
        raise FAError(st, "fa_decode")
    return out, lse


def flash_attn_with_kvcache(q, k_cache, v_cache, cache_seqlens, softmax_scale=None, causal=False):
    """decode() returning O only (inference: no gradient)."""
    return decode(q, k_cache, v_cache, cache_seqlens, softmax_scale, causal)[0]


# ------------------------------------------------------------ status, hooks

def check_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word
    of the current device (or of the stream's device when one is given)."""
    import torch
    device = stream.device if stream is not None else torch.cuda.current_device()
    with torch.cuda.device(device):
        return int(library().fa_check_device_status(_stream_ptr(stream, device)))


def profile_bwd_events(begin=None, end=None) -> None:
    """Bracket the dK/dV kernel of this thread's following backward calls with
    two torch.cuda.Event objects (enable_timing=True); None, None stops."""
    for ev in (begin, end):
        if ev is not None and not ev.cuda_event:
            ev.record()  # torch creates the underlying CUDA event on its first record
    st = library().fa_profile_bwd_events(None if begin is None else ctypes.c_void_p(begin.cuda_event),
                                         None if end is None else ctypes.c_void_p(end.cuda_event))
    if st != FA_OK:
        raise FAError(st, "fa_profile_bwd_events")


def selftest_bounded_wait(which: int, limit_ms: int = 50, stream=None) -> None:
    """Launch the failure-detection self-test kernel (described in include/fa.h)
    on the current device."""
    st = library().fa_selftest_bounded_wait(int(which), int(limit_ms), _stream_ptr(stream))
    if st != FA_OK:
        raise FAError(st, "fa_selftest_bounded_wait")


# ------------------------------------------------------------------ autograd

_fns = {}


def _autograd_functions():
    if _fns:
        return _fns
    import torch

    def draw_seed():
        # A fresh 64-bit seed per call from torch's host generator, kept for
        # the backward, which regenerates the same mask.
        return int(torch.randint(0, 2 ** 62, (1,), dtype=torch.int64).item())

    class _FlashAttention(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, dropout_p, softmax_scale, causal):
            seed = draw_seed() if dropout_p else None
            o, lse = forward(q, k, v, softmax_scale, causal, dropout_p=dropout_p, seed=seed)
            ctx.save_for_backward(q, k, v, o, lse)
            ctx.args = (softmax_scale, causal, dropout_p, seed)
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse = ctx.saved_tensors
            scale, causal, p, seed = ctx.args
            dq, dk, dv = backward(q, k, v, o, _dense_last(do), lse, scale, causal, dropout_p=p, seed=seed)
            return dq, dk, dv, None, None, None

    class _FlashAttentionQKVPacked(torch.autograd.Function):
        @staticmethod
        def forward(ctx, qkv, dropout_p, softmax_scale, causal):
            seed = draw_seed() if dropout_p else None
            q, k, v = qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2]
            o, lse = forward(q, k, v, softmax_scale, causal, dropout_p=dropout_p, seed=seed)
            ctx.save_for_backward(qkv, o, lse)
            ctx.args = (softmax_scale, causal, dropout_p, seed)
            return o

        @staticmethod
        def backward(ctx, do):
            qkv, o, lse = ctx.saved_tensors
            scale, causal, p, seed = ctx.args
            dqkv = torch.empty_like(qkv, memory_format=torch.contiguous_format)
            backward(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], o, _dense_last(do), lse, scale, causal,
                     dqkv[:, :, 0], dqkv[:, :, 1], dqkv[:, :, 2], dropout_p=p, seed=seed)
            return dqkv, None, None, None

    class _FlashAttentionVarlen(torch.autograd.Function):
        @staticmethod
        def forward(ctx, q, k, v, cu_seqlens, max_seqlen, dropout_p, softmax_scale, causal):
            seed = draw_seed() if dropout_p else None
            o, lse = varlen_forward(q, k, v, cu_seqlens, max_seqlen, softmax_scale, causal, dropout_p=dropout_p,
                                    seed=seed)
            ctx.save_for_backward(q, k, v, o, lse, cu_seqlens)
            ctx.args = (max_seqlen, softmax_scale, causal, dropout_p, seed)
            return o

        @staticmethod
        def backward(ctx, do):
            q, k, v, o, lse, cu = ctx.saved_tensors
            max_seqlen, scale, causal, p, seed = ctx.args
            dq, dk, dv = varlen_backward(q, k, v, o, _dense_last(do), lse, cu, max_seqlen, scale, causal,
                                         dropout_p=p, seed=seed)
            return dq, dk, dv, None, None, None, None, None

    _fns.update(plain=_FlashAttention, packed=_FlashAttentionQKVPacked, varlen=_FlashAttentionVarlen)
    return _fns


def _dense_last(t):
    # The upstream gradient may be any view (even expanded, stride 0): the
    # kernels need a contiguous head_dim and strides that are multiples of 8.
    ok = t.stride(-1) == 1 and all(n == 1 or (s % 8 == 0 and s > 0) for n, s in zip(t.shape[:-1], t.stride()[:-1]))
    return t if ok else t.contiguous()


def flash_attn_func(q, k, v, dropout_p=0.0, softmax_scale=None, causal=False):
    """Differentiable exact attention on [B, N, H, d] fp16/bf16 CUDA tensors,
    with the argument order the lab write-up's §4.2 gives flash_attn_func
    (dropout on P when dropout_p > 0; a fresh seed per call)."""
    return _autograd_functions()["plain"].apply(q, k, v, dropout_p, softmax_scale, causal)


def flash_attn_qkvpacked_func(qkv, dropout_p=0.0, softmax_scale=None, causal=False):
    """Differentiable exact attention on one packed [B, N, 3, H, d] tensor (q,
    k, v along dim 2), read in place; its gradient comes back packed."""
    if qkv.dim() != 5 or qkv.shape[2] != 3:
        raise ValueError(f"qkv must be [batch, seqlen, 3, heads, head_dim], got {tuple(qkv.shape)}")
    return _autograd_functions()["packed"].apply(qkv, dropout_p, softmax_scale, causal)


def flash_attn_varlen_func(q, k, v, cu_seqlens, max_seqlen, dropout_p=0.0, softmax_scale=None, causal=False):
    """Differentiable exact attention over a variable-length batch packed
    without padding ([total, H, d] tensors, int32 row offsets cu_seqlens)."""
    return _autograd_functions()["varlen"].apply(q, k, v, cu_seqlens, max_seqlen, dropout_p, softmax_scale, causal)

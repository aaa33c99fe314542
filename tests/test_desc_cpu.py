"""Host-side checks of the descriptor calls (fa_fwd_ex, fa_bwd_ex, fa_decode),
CPU only. Every call passes misaligned (8-byte) pointers as a second guard, so
that even a check that wrongly passed would stop at the pointer check, never
at a launch; each test asserts, from fa_last_error_detail(), that the check it
targets is the one that fired."""

import ctypes

import pytest

import exact_attention_119_b200 as fa


@pytest.fixture(scope="module")
def lib():
    from exact_attention_119_b200 import build
    build.build()
    return fa.library()


BAD = ctypes.c_void_p(8)   # misaligned: rejected before any launch


def desc(**kw):
    x = fa.FaDesc()
    x.B, x.N, x.H, x.d = kw.get("B", 2), kw.get("N", 256), kw.get("H", 4), kw.get("d", 64)
    x.softmax_scale = kw.get("scale", 0.125)
    x.causal = kw.get("causal", 0)
    x.dtype = kw.get("dtype", 1)
    for name in ("q", "k", "v", "o", "do", "dq", "dk", "dv"):
        if name in kw:
            setattr(x, "stride_" + name, fa.FaStrides(*kw[name]))
    x.cu_seqlens = kw.get("cu", None)
    x.total = kw.get("total", 0)
    x.dropout_p = kw.get("p", 0.0)
    x.seed = kw.get("seed", 0)
    return x


def fwd(lib, d):
    return lib.fa_fwd_ex(ctypes.byref(d), BAD, BAD, BAD, BAD, BAD, None)


def bwd(lib, d):
    return lib.fa_bwd_ex(ctypes.byref(d), BAD, BAD, BAD, BAD, BAD, BAD, BAD, BAD, BAD, ctypes.c_void_p(16), 1 << 30,
                         None)


def test_valid_descriptor_reaches_the_pointer_check(lib):
    assert fwd(lib, desc()) == 1
    assert "aligned" in fa.last_error_detail()
    assert bwd(lib, desc(q=(256 * 3 * 4 * 64, 3 * 4 * 64, 64))) == 1   # a packed-QKV q view is fine
    assert "aligned" in fa.last_error_detail()


@pytest.mark.parametrize("strides,what", [
    ((256 * 4 * 64, 4 * 64, 63), "q strides"),     # head stride not a multiple of 8
    ((256 * 4 * 64, 4 * 60, 64), "q strides"),     # row stride 240: fine (multiple of 8) -> see below
    ((0, 4 * 64, 64), "q strides"),                # batch stride 0 with B = 2
    ((256 * 4 * 64, 0, 64), "q strides"),          # row stride 0
    ((256 * 4 * 64, 4 * 64, 1 << 37), "q strides"),  # beyond 2^36
])
def test_bad_strides(lib, strides, what):
    st = fwd(lib, desc(q=strides))
    if strides[1] == 240:
        assert st == 1 and "aligned" in fa.last_error_detail()   # a legal (if overlapping) view
    else:
        assert st == 1 and what in fa.last_error_detail()


def test_batch_stride_zero_allowed_for_one_batch(lib):
    assert fwd(lib, desc(B=1, q=(0, 4 * 64, 64))) == 1
    assert "aligned" in fa.last_error_detail()


def test_other_descriptor_checks(lib):
    assert fwd(lib, desc(d=100)) == 2 and "head_dim" in fa.last_error_detail()
    assert fwd(lib, desc(d=136)) == 2
    assert fwd(lib, desc(B=1000, H=100)) == 2 and "65535" in fa.last_error_detail()
    assert fwd(lib, desc(p=1.0)) == 1 and "dropout_p" in fa.last_error_detail()
    assert fwd(lib, desc(p=-0.1)) == 1 and "dropout_p" in fa.last_error_detail()
    assert fwd(lib, desc(causal=3)) == 1 and "causal" in fa.last_error_detail()
    assert fwd(lib, desc(dtype=5)) == 1 and "dtype" in fa.last_error_detail()
    assert lib.fa_fwd_ex(None, BAD, BAD, BAD, BAD, BAD, None) == 1 and "NULL" in fa.last_error_detail()


def test_varlen_checks(lib):
    assert fwd(lib, desc(cu=ctypes.c_void_p(18).value, total=10)) == 1
    assert "cu_seqlens" in fa.last_error_detail()
    assert fwd(lib, desc(cu=ctypes.c_void_p(16).value, total=0)) == 1
    assert "total" in fa.last_error_detail()
    assert fwd(lib, desc(cu=ctypes.c_void_p(16).value, total=1000)) == 1
    assert "aligned" in fa.last_error_detail()


def test_workspace_sizes(lib):
    d = desc(B=2, N=300, H=3, d=40)
    assert lib.fa_bwd_ex_workspace_size(ctypes.byref(d)) == lib.fa_bwd_workspace_size(2, 300, 3, 64, 0)
    assert lib.fa_bwd_ex_workspace_size(ctypes.byref(desc(d=12))) == 0
    assert fa.decode_workspace_size(8, 1, 32, 128, 8192) > 0
    assert fa.decode_workspace_size(8, 9, 32, 128, 8192) == 0     # more than 8 new rows
    assert fa.decode_workspace_size(8, 1, 32, 100, 8192) == 0


def test_decode_checks(lib):
    lens = ctypes.c_void_p(16)
    ws = ctypes.c_void_p(16)
    args = lambda B=2, Nq=1, H=2, d=64, N=128, scale=0.125, causal=0, dtype=1: (
        BAD, BAD, BAD, lens, BAD, BAD, ws, 1 << 30, B, Nq, H, d, N, scale, causal, dtype, None)
    assert lib.fa_decode(*args(Nq=9)) == 2 and "8 query rows" in fa.last_error_detail()
    assert lib.fa_decode(*args(d=72 + 1)) == 2
    assert lib.fa_decode(*args(scale=0.0)) == 1 and "softmax_scale" in fa.last_error_detail()
    assert lib.fa_decode(*args()) == 1 and "aligned" in fa.last_error_detail()

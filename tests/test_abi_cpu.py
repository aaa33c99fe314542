"""The C ABI library loads, exports what include/fa.h declares, and rejects bad
arguments on the host before touching the GPU (CPU only; no compute calls)."""

import ctypes
import os
import re

import pytest

import exact_attention_119_b200 as fa

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"FA_API\s+[\w\s\*]+?\b(fa_\w+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from exact_attention_119_b200 import build
    build.build()
    return fa.library()


def test_header_declares_the_boundary():
    names = declared_functions()
    for want in ("fa_fwd", "fa_bwd", "fa_bwd_workspace_size", "fa_check_device_status", "fa_status_string"):
        assert want in names


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    assert fa.status_string(0) == "FA_OK"
    assert fa.status_string(4) == "FA_ERR_DEVICE_TIMEOUT"
    assert fa.status_string(99) == "FA_ERR_UNKNOWN"


def _fwd(lib, ptr=16, B=1, N=8, H=1, d=64, scale=0.125, causal=0, dtype=0):
    p = ctypes.c_void_p(ptr)
    return lib.fa_fwd(p, p, p, p, p, B, N, H, d, scale, causal, dtype, None)


def test_fwd_rejects_bad_arguments_before_launch(lib):
    assert _fwd(lib, ptr=0) == 1                 # null pointer
    assert _fwd(lib, ptr=8) == 1                 # misaligned
    assert _fwd(lib, N=0) == 1
    assert _fwd(lib, B=-1) == 1
    assert _fwd(lib, scale=0.0) == 1
    assert _fwd(lib, scale=float("nan")) == 1
    assert _fwd(lib, scale=-1.0) == 1
    assert _fwd(lib, causal=2) == 1
    assert _fwd(lib, dtype=7) == 1
    assert _fwd(lib, d=12) == 2                  # unsupported head sizes (not a multiple of 8, > 128)
    assert _fwd(lib, d=136) == 2
    assert _fwd(lib, d=256) == 2
    assert _fwd(lib, B=1 << 10, N=1 << 12, H=8, d=128) == 2   # >= 2^31 elements


def test_workspace_size(lib):
    assert fa.bwd_workspace_size(1, 1, 1, 64) > 0
    assert fa.bwd_workspace_size(0, 1, 1, 64) == 0
    assert fa.bwd_workspace_size(1, 1, 1, 84) == 0
    assert fa.bwd_workspace_size(1, 1, 1, 80) == fa.bwd_workspace_size(1, 1, 1, 128)
    small = fa.bwd_workspace_size(1, 128, 1, 64)
    assert fa.bwd_workspace_size(1, 256, 1, 64) > small
    assert fa.bwd_workspace_size(2, 128, 1, 64) > small


def test_bwd_rejects_bad_workspace(lib):
    p = ctypes.c_void_p(16)
    args = [p] * 9
    need = lib.fa_bwd_workspace_size(1, 128, 1, 64, 0)
    assert lib.fa_bwd(*args, ctypes.c_void_p(0), need, 1, 128, 1, 64, 0.125, 0, 0, None) == 5
    assert lib.fa_bwd(*args, p, need - 1, 1, 128, 1, 64, 0.125, 0, 0, None) == 5
    assert lib.fa_bwd(*args, p, need, 1, 128, 1, 20, 0.125, 0, 0, None) == 2


def test_python_binding_rejects_fp32():
    import torch
    x = torch.zeros(1, 4, 1, 64)
    with pytest.raises(TypeError):
        fa.forward(x, x, x)


def test_last_error_detail_names_the_failed_check(lib):
    assert _fwd(lib, scale=0.0) == 1
    assert "softmax_scale" in fa.last_error_detail()
    assert _fwd(lib, d=100) == 2
    assert "head_dim" in fa.last_error_detail()
    assert _fwd(lib, ptr=8) == 1
    assert "aligned" in fa.last_error_detail()


def test_profile_hook_needs_both_events_or_neither(lib):
    assert lib.fa_profile_bwd_events(ctypes.c_void_p(16), None) == 1
    assert lib.fa_profile_bwd_events(None, ctypes.c_void_p(16)) == 1
    assert lib.fa_profile_bwd_events(None, None) == 0


class _OnDevice:
    def __init__(self, device):
        self.device = device


def test_binding_rejects_tensors_and_streams_on_another_device():
    # forward/backward run on q's device; anything else the call would touch
    # (lse, outputs, workspace, stream) must be on that device too.
    import torch
    d0, d1 = torch.device("cuda", 0), torch.device("cuda", 1)
    fa.check_same_device(d0, lse=_OnDevice(d0), stream=_OnDevice(d0), workspace=None)
    with pytest.raises(ValueError, match="lse"):
        fa.check_same_device(d0, lse=_OnDevice(d1))
    with pytest.raises(ValueError, match="stream"):
        fa.check_same_device(d0, lse=_OnDevice(d0), stream=_OnDevice(d1))
    with pytest.raises(ValueError, match="workspace"):
        fa.check_same_device(d1, workspace=_OnDevice(d0))

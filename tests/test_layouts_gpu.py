"""Layouts on a B200 against the fp64 oracle: packed QKV, head-major and other
strided views, outputs inside larger buffers, head sizes that are multiples of
8 up to 128, and variable-length batches packed without padding.

Every case compares the CUDA path (through the C ABI's fa_fwd_ex / fa_bwd_ex)
element by element with the oracle on the same seeded inputs: O max-abs, LSE
max-abs, dQ/dK/dV relative Frobenius error, at the tolerances the other tests
use.
"""

import math

import numpy as np
import pytest

from exact_attention_119_b200 import inputs
from helpers import GRAD_REL_TOL, LSE_TOL, O_TOL, Case, max_abs, rel_fro
from oracle import attention_backward, attention_backward_varlen, attention_forward, attention_forward_varlen

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_attention_119_b200 as fa
    fa.library()


def np64(t):
    return t.double().cpu().numpy()


def check_fwd(o, lse, case):
    ro, rl = attention_forward(case.f64["q"], case.f64["k"], case.f64["v"], case.scale, case.causal)
    assert max_abs(np64(o), ro) <= O_TOL[case.dtype], case
    assert max_abs(np64(lse), rl) <= LSE_TOL, case


def check_grads(grads, case):
    ref = attention_backward(case.f64["q"], case.f64["k"], case.f64["v"], case.f64["do"], case.scale,
                             case.causal)[:3]
    for g, r in zip(grads, ref):
        g = np64(g)
        assert np.isfinite(g).all(), case
        assert rel_fro(g, r) <= GRAD_REL_TOL, case


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H,d,dtype", [(2, 2048, 12, 64, "fp16"), (1, 700, 4, 128, "bf16")])
def test_qkvpacked(B, N, H, d, dtype, causal):
    # One [B, N, 3, H, d] tensor read in place (the shape of the PyTorch
    # comparison page), gradient returned packed through autograd.
    import exact_attention_119_b200 as fa
    case = Case(B, N, H, d, dtype, causal, seed=41)
    qkv = torch.stack([case.torch(n) for n in ("q", "k", "v")], dim=2).contiguous().requires_grad_(True)
    o = fa.flash_attn_qkvpacked_func(qkv, 0.0, case.scale, causal)
    o.backward(case.torch("do"))
    assert fa.check_device_status() == 0
    _, lse = fa.forward(qkv[:, :, 0].detach(), qkv[:, :, 1].detach(), qkv[:, :, 2].detach(), case.scale, causal)
    check_fwd(o.detach(), lse, case)
    g = qkv.grad
    assert g.shape == qkv.shape
    check_grads((g[:, :, 0], g[:, :, 1], g[:, :, 2]), case)


@pytest.mark.parametrize("causal", [False, True])
def test_head_major_inputs_and_strided_outputs(causal):
    # q, k, v, dO stored [B, H, N, d] (PyTorch's attention layout) and passed
    # as [B, N, H, d] views; O, dQ, dK, dV written into slices of larger
    # buffers whose other columns keep their fill.
    import exact_attention_119_b200 as fa
    B, N, H, d = 2, 520, 3, 64
    case = Case(B, N, H, d, "bf16", causal, seed=43)
    hm = {n: case.torch(n).transpose(1, 2).contiguous().transpose(1, 2) for n in ("q", "k", "v", "do")}
    assert hm["q"].stride() == (H * N * d, d, N * d, 1)
    bufs = [torch.full((B, N, H, d + 16), 5.0, dtype=torch.bfloat16, device="cuda") for _ in range(4)]
    out, dq, dk, dv = (b[..., 8:8 + d] for b in bufs)
    o, lse = fa.forward(hm["q"], hm["k"], hm["v"], case.scale, causal, out=out)
    grads = fa.backward(hm["q"], hm["k"], hm["v"], o, hm["do"], lse, case.scale, causal, dq, dk, dv)
    assert fa.check_device_status() == 0
    check_fwd(o, lse, case)
    check_grads(grads, case)
    for b in bufs:
        assert torch.all(b[..., :8] == 5.0) and torch.all(b[..., 8 + d:] == 5.0)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(128, "bf16"), (64, "fp16")])
def test_head_major_outputs(d, dtype, causal):
    # O, dQ, dK, dV written into [B, H, N, d] storage through [B, N, H, d]
    # views: the output tensor maps are head-major, and N = 300 leaves a
    # ragged last tile whose rows past N must not be written.
    import exact_attention_119_b200 as fa
    B, N, H = 2, 300, 3
    case = Case(B, N, H, d, dtype, causal, seed=47)
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    store = [torch.full((B, H, N + 8, d), 7.0, dtype=q.dtype, device="cuda") for _ in range(4)]
    out, dq, dk, dv = (t[:, :, :N].transpose(1, 2) for t in store)
    assert out.stride() == (H * (N + 8) * d, d, (N + 8) * d, 1)
    o, lse = fa.forward(q, k, v, case.scale, causal, out=out)
    grads = fa.backward(q, k, v, o, do, lse, case.scale, causal, dq, dk, dv)
    assert fa.check_device_status() == 0
    check_fwd(o, lse, case)
    check_grads(grads, case)
    for t in store:
        assert torch.all(t[:, :, N:] == 7.0)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d", [8, 16, 32, 40, 48, 72, 80, 96, 112, 120])
def test_head_sizes(d, causal):
    # Head sizes between the kernels' 64- and 128-column tiles: the tensor
    # maps read zeros past d, and nothing is written past d (canary columns).
    import exact_attention_119_b200 as fa
    dtype = "fp16" if d % 16 else "bf16"
    case = Case(2, 333, 3, d, dtype, causal, seed=d)
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    tdt = q.dtype
    bufs = [torch.full((2, 333, 3, d + 8), 3.0, dtype=tdt, device="cuda") for _ in range(4)]
    out, dq, dk, dv = (b[..., :d] for b in bufs)
    o, lse = fa.forward(q, k, v, case.scale, causal, out=out)
    grads = fa.backward(q, k, v, o, do, lse, case.scale, causal, dq, dk, dv)
    assert fa.check_device_status() == 0
    check_fwd(o, lse, case)
    check_grads(grads, case)
    for b in bufs:
        assert torch.all(b[..., d:] == 3.0)


def varlen_case(lens, H, d, dtype, causal, seed):
    total = int(sum(lens))
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    bits = {n: inputs.make_tensor_bits((total, H, d), dtype, seed, s) for n, s in
            (("q", 0), ("k", 1), ("v", 2), ("do", 3))}
    t = {n: inputs.bits_to_torch(b, dtype).cuda() for n, b in bits.items()}
    f = {n: inputs.bits_to_f64(b, dtype) for n, b in bits.items()}
    return cu, t, f


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16"), (40, "fp16")])
def test_varlen_matches_oracle(d, dtype, causal):
    import exact_attention_119_b200 as fa
    lens = [1, 127, 128, 300, 0, 1000, 513, 2]
    H = 3
    cu, t, f = varlen_case(lens, H, d, dtype, causal, seed=51)
    cu_t = torch.from_numpy(cu).cuda()
    scale = 1.0 / math.sqrt(d)
    o, lse = fa.varlen_forward(t["q"], t["k"], t["v"], cu_t, max(lens), scale, causal)
    dq, dk, dv = fa.varlen_backward(t["q"], t["k"], t["v"], o, t["do"], lse, cu_t, max(lens), scale, causal)
    assert fa.check_device_status() == 0
    ro, rl = attention_forward_varlen(f["q"], f["k"], f["v"], cu, scale, causal)
    assert max_abs(np64(o), ro) <= O_TOL[dtype]
    assert max_abs(np64(lse), rl) <= LSE_TOL
    ref = attention_backward_varlen(f["q"], f["k"], f["v"], f["do"], cu, scale, causal)
    for name, g, r in zip(("dq", "dk", "dv"), (dq, dk, dv), ref):
        g = np64(g)
        assert np.isfinite(g).all(), name
        # per sequence with keys: a one-row sequence has dQ = dK = 0 exactly
        for a, e in zip(cu[:-1], cu[1:]):
            if e - a >= 2:
                assert rel_fro(g[a:e], r[a:e]) <= GRAD_REL_TOL, (name, a, e)
            else:
                assert np.abs(g[a:e] - r[a:e]).max(initial=0.0) <= 1e-3, (name, a, e)


def test_varlen_autograd_and_max_seqlen_bound():
    # flash_attn_varlen_func through autograd equals the direct calls; a
    # max_seqlen above every length changes nothing.
    import exact_attention_119_b200 as fa
    lens = [200, 57, 384]
    cu, t, f = varlen_case(lens, 2, 64, "bf16", True, seed=53)
    cu_t = torch.from_numpy(cu).cuda()
    q, k, v = (t[n].clone().requires_grad_(True) for n in ("q", "k", "v"))
    y = fa.flash_attn_varlen_func(q, k, v, cu_t, max(lens), 0.0, 0.125, True)
    y.backward(t["do"])
    o, lse = fa.varlen_forward(t["q"], t["k"], t["v"], cu_t, 1000, 0.125, True)
    grads = fa.varlen_backward(t["q"], t["k"], t["v"], o, t["do"], lse, cu_t, 1000, 0.125, True)
    torch.cuda.synchronize()
    assert fa.check_device_status() == 0
    ro, _ = attention_forward_varlen(f["q"], f["k"], f["v"], cu, 0.125, True)
    assert max_abs(np64(y.detach()), ro) <= O_TOL["bf16"]
    assert max_abs(np64(o), ro) <= O_TOL["bf16"]
    ref = attention_backward_varlen(f["q"], f["k"], f["v"], f["do"], cu, 0.125, True)
    for a, b, r in zip((q.grad, k.grad, v.grad), grads, ref):
        assert rel_fro(np64(a), r) <= GRAD_REL_TOL
        assert rel_fro(np64(b), r) <= GRAD_REL_TOL


def test_varlen_long_sequences_sampled():
    # A long packed batch (two 4096-row sequences and a ragged one) at the
    # d = 128 bf16 decoder setting; full forward parity, backward on one head.
    import exact_attention_119_b200 as fa
    lens = [4096, 1500, 4096]
    cu, t, f = varlen_case(lens, 4, 128, "bf16", True, seed=55)
    cu_t = torch.from_numpy(cu).cuda()
    scale = 1.0 / math.sqrt(128)
    o, lse = fa.varlen_forward(t["q"], t["k"], t["v"], cu_t, 4096, scale, True)
    dq, dk, dv = fa.varlen_backward(t["q"], t["k"], t["v"], o, t["do"], lse, cu_t, 4096, scale, True)
    assert fa.check_device_status() == 0
    ro, rl = attention_forward_varlen(f["q"], f["k"], f["v"], cu, scale, True)
    assert max_abs(np64(o), ro) <= O_TOL["bf16"]
    assert max_abs(np64(lse), rl) <= LSE_TOL
    h = 3
    one = {n: f[n][:, h:h + 1] for n in f}
    ref = attention_backward_varlen(one["q"], one["k"], one["v"], one["do"], cu, scale, True)
    for g, r in zip((dq, dk, dv), ref):
        assert rel_fro(np64(g)[:, h:h + 1], r) <= GRAD_REL_TOL


def test_varlen_rejects_bad_offsets_tensor():
    import exact_attention_119_b200 as fa
    q = torch.zeros(10, 2, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(ValueError):
        fa.varlen_forward(q, q, q, torch.tensor([0, 10], dtype=torch.int64, device="cuda"), 10)

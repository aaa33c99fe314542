"""Dropout on a B200 (fa_fwd_ex / fa_bwd_ex with dropout_p > 0) against the
fp64 oracle, which draws the same keep mask from its own Philox4x32-10.

The mask is integer work (a 32-bit word compared with floor(p * 2^32)), so it
is checked bit for bit: with q = 0 every probability of a row is 1/N, and with
V = the identity (d = N = 128) O[i, j] = keep(i, j) / (N (1 - p)), which shows
every mask bit in the output. O is then checked element by element against
the oracle within the O tolerance scaled by 1/(1 - p) (the kept values are
scaled by it), LSE within the usual tolerance (dropout does not touch it), and
dQ, dK, dV by relative Frobenius error."""

import math

import numpy as np
import pytest

from exact_attention_119_b200 import inputs
from helpers import GRAD_REL_TOL, LSE_TOL, O_TOL, Case, max_abs, rel_fro
from oracle import (attention_backward_dropout, attention_forward_dropout, attention_forward_varlen,
                    dropout_keep)

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


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_mask_bit_exact(p, dtype):
    import exact_attention_119_b200 as fa
    B, N, H, d = 2, 128, 3, 128
    tdt = torch.float16 if dtype == "fp16" else torch.bfloat16
    q = torch.zeros(B, N, H, d, dtype=tdt, device="cuda")
    k = torch.randn(B, N, H, d, dtype=tdt, device="cuda")
    v = torch.eye(N, dtype=tdt, device="cuda")[None, :, None, :].expand(B, N, H, d).contiguous()
    seed, offset = 0x1234_5678_9ABC, 17
    o, _ = fa.forward(q, k, v, 0.1, False, dropout_p=p, seed=seed, offset=offset)
    assert fa.check_device_status() == 0
    got = np64(o) > 0
    for b in range(B):
        for h in range(H):
            want = dropout_keep(b, h, H, N, N, p, seed, offset)
            assert np.array_equal(got[b, :, h, :], want), (b, h)
    kept = np64(o)[got]
    np.testing.assert_allclose(kept, 1.0 / (N * (1 - p)), rtol=2 ** -7)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("B,N,H,d,dtype,p", [(1, 300, 2, 64, "fp16", 0.2), (2, 1000, 3, 128, "bf16", 0.1),
                                              (1, 257, 2, 40, "fp16", 0.5)])
def test_forward_backward_match_oracle(B, N, H, d, dtype, p, causal):
    import exact_attention_119_b200 as fa
    case = Case(B, N, H, d, dtype, causal, seed=61)
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    seed, offset = 2024, 3
    o, lse = fa.forward(q, k, v, case.scale, causal, dropout_p=p, seed=seed, offset=offset)
    grads = fa.backward(q, k, v, o, do, lse, case.scale, causal, dropout_p=p, seed=seed, offset=offset)
    assert fa.check_device_status() == 0
    ro, rl = attention_forward_dropout(case.f64["q"], case.f64["k"], case.f64["v"], case.scale, causal, p, seed,
                                       offset)
    assert max_abs(np64(o), ro) <= O_TOL[dtype] / (1 - p)
    assert max_abs(np64(lse), rl) <= LSE_TOL
    ref = attention_backward_dropout(case.f64["q"], case.f64["k"], case.f64["v"], case.f64["do"], case.scale,
                                     causal, p, seed, offset)
    for g, r in zip(grads, ref):
        g = np64(g)
        assert np.isfinite(g).all()
        assert rel_fro(g, r) <= GRAD_REL_TOL


def test_varlen_with_dropout():
    import exact_attention_119_b200 as fa
    lens = [300, 0, 129, 64]
    total, H, d, dtype, p = sum(lens), 2, 64, "bf16", 0.25
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    bits = {n: inputs.make_tensor_bits((total, H, d), dtype, 71, s) for n, s in (("q", 0), ("k", 1), ("v", 2))}
    t = {n: inputs.bits_to_torch(b, dtype).cuda() for n, b in bits.items()}
    f = {n: inputs.bits_to_f64(b, dtype) for n, b in bits.items()}
    o, lse = fa.varlen_forward(t["q"], t["k"], t["v"], torch.from_numpy(cu).cuda(), max(lens), 0.125, True,
                               dropout_p=p, seed=5, offset=1)
    assert fa.check_device_status() == 0
    ro, rl = attention_forward_varlen(f["q"], f["k"], f["v"], cu, 0.125, True, dropout=(p, 5, 1))
    assert max_abs(np64(o), ro) <= O_TOL[dtype] / (1 - p)
    assert max_abs(np64(lse), rl) <= LSE_TOL


def test_seed_decides_the_mask_and_autograd_runs():
    import exact_attention_119_b200 as fa
    case = Case(1, 200, 2, 64, "bf16", False, seed=81)
    q, k, v = (case.torch(n) for n in ("q", "k", "v"))
    a1, _ = fa.forward(q, k, v, None, False, dropout_p=0.3, seed=1)
    a2, _ = fa.forward(q, k, v, None, False, dropout_p=0.3, seed=1)
    b1, _ = fa.forward(q, k, v, None, False, dropout_p=0.3, seed=2)
    assert torch.equal(a1, a2) and not torch.equal(a1, b1)
    qr, kr, vr = (x.clone().requires_grad_(True) for x in (q, k, v))
    torch.manual_seed(0)
    y1 = fa.flash_attn_func(qr, kr, vr, 0.3)
    y1.float().sum().backward()
    torch.manual_seed(0)
    y2 = fa.flash_attn_func(q, k, v, 0.3)
    assert torch.equal(y1.detach(), y2)
    assert all(torch.isfinite(g).all() for g in (qr.grad, kr.grad, vr.grad))
    with pytest.raises(ValueError):
        fa.forward(q, k, v, None, False, dropout_p=0.3)   # no seed: the backward could not redraw the mask

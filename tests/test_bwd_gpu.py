"""Backward parity on a B200: fa_bwd (through the C ABI, fed by fa_fwd's O and
LSE) against the fp64 oracle's dQ, dK, dV, by relative Frobenius error."""

import numpy as np
import pytest

from helpers import GRAD_REL_TOL, Case, rel_fro
from oracle import attention_backward

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_attention_119_b200 as fa
    fa.library()


def run_bwd(case):
    import exact_attention_119_b200 as fa
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, case.scale, case.causal)
    dq, dk, dv = fa.backward(q, k, v, o, do, lse, case.scale, case.causal)
    assert fa.check_device_status() == 0
    return [t.double().cpu().numpy() for t in (dq, dk, dv)]


def check(case, heads=None):
    got = run_bwd(case)
    ref = attention_backward(case.f64["q"], case.f64["k"], case.f64["v"], case.f64["do"], case.scale,
                             case.causal, heads=heads)[:3]
    pairs = heads or [(b, h) for b in range(case.B) for h in range(case.H)]
    dos = np.stack([case.f64["do"][b, :, h] for b, h in pairs])
    errs = []
    for name, g, r in zip(("dq", "dk", "dv"), got, ref):
        assert np.isfinite(g).all(), (case, name)
        gs = np.stack([g[b, :, h] for b, h in pairs])
        rs = np.stack([r[b, :, h] for b, h in pairs])
        if np.linalg.norm(rs) == 0.0:
            # Degenerate case (e.g. N = 1: P = 1, so dS = 0 and dQ = dK = 0
            # exactly): no relative error exists; the GPU's rounding residue
            # must be negligible next to the upstream gradient.
            e = float(np.linalg.norm(gs) / np.linalg.norm(dos))
            assert e <= 1e-4, (case, name, e)
        else:
            e = rel_fro(gs, rs)
            assert e <= GRAD_REL_TOL, (case, name, e)
        errs.append(e)
    return errs


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
def test_small(d, dtype, causal):
    check(Case(1, 128, 2, d, dtype, causal))
    check(Case(2, 384, 3, d, dtype, causal, seed=1))


@pytest.mark.parametrize("N", [1, 2, 7, 127, 129, 255, 257, 300, 1000])
@pytest.mark.parametrize("causal", [False, True])
def test_ragged_lengths(N, causal):
    check(Case(2, N, 2, 64, "fp16", causal, seed=N))
    check(Case(1, N, 3, 128, "bf16", causal, seed=N + 1))


def test_tiny_config():
    check(Case(1, 128, 2, 64, "fp16", False))


def test_p4_shape_config():
    check(Case(2, 2048, 12, 64, "fp16", False))


@pytest.mark.parametrize("B,H", [(4, 8), (1, 32)])
def test_decoder_and_llama_layer_configs(B, H):
    check(Case(B, 4096, H, 128, "bf16", True))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [512, 2048])
def test_sweep_short(N, causal):
    check(Case(16384 // N, N, 16, 128, "bf16", causal))


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N", [8192, 16384, 32768])
def test_sweep_long_sampled_heads(N, causal):
    B = max(1, 16384 // N)
    check(Case(B, N, 16, 128, "bf16", causal), heads=[(0, 0), (B - 1, 15)])


@pytest.mark.parametrize("causal", [False, True])
def test_stability_large_logits(causal):
    check(Case(2, 8192, 16, 128, "bf16", causal, sigma_qk=3.0), heads=[(0, 0), (1, 15)])


def test_deterministic():
    import exact_attention_119_b200 as fa
    case = Case(2, 1500, 4, 128, "bf16", True, seed=9)
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, case.scale, True)
    a = fa.backward(q, k, v, o, do, lse, case.scale, True)
    b = fa.backward(q, k, v, o, do, lse, case.scale, True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_workspace_reuse_and_no_overrun():
    # A caller-provided workspace is reused across calls without zeroing, and
    # the outputs keep a canary past their last row.
    import exact_attention_119_b200 as fa
    case = Case(1, 200, 2, 64, "fp16", False, seed=4)
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, case.scale, False)
    need = fa.bwd_workspace_size(1, 200, 2, 64, False)
    ws = torch.full((need,), 0x7F, dtype=torch.uint8, device="cuda")
    n = 200 * 2 * 64
    bufs = [torch.full((2 * n,), 3.0, dtype=torch.float16, device="cuda") for _ in range(3)]
    views = [b[:n].view(1, 200, 2, 64) for b in bufs]
    r1 = [x.clone() for x in fa.backward(q, k, v, o, do, lse, case.scale, False, *views, workspace=ws)]
    r2 = fa.backward(q, k, v, o, do, lse, case.scale, False, *views, workspace=ws)
    torch.cuda.synchronize()
    for x, y in zip(r1, r2):
        assert torch.equal(x, y)
    for b in bufs:
        assert torch.all(b[n:] == 3.0)


@pytest.mark.parametrize("causal", [False, True])
def test_autograd_wrapper_matches_direct_calls(causal):
    # flash_attn_func (torch.autograd.Function over fa_fwd / fa_bwd) returns
    # exactly what the direct calls return; the backward is deterministic.
    import exact_attention_119_b200 as fa
    case = Case(1, 300, 2, 64, "fp16", causal, seed=3)
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    qr, kr, vr = (t.clone().requires_grad_(True) for t in (q, k, v))
    y = fa.flash_attn_func(qr, kr, vr, 0.0, case.scale, causal)
    y.backward(do)
    o, lse = fa.forward(q, k, v, case.scale, causal)
    dq, dk, dv = fa.backward(q, k, v, o, do, lse, case.scale, causal)
    torch.cuda.synchronize()
    assert torch.equal(y.detach(), o)
    for got, want in ((qr.grad, dq), (kr.grad, dk), (vr.grad, dv)):
        assert torch.equal(got, want)


def _workspace_d(ws, B, N, H):
    """D = rowsum(dO o O) as fa_bwd left it in the workspace: [B*H, N_pad]
    fp32 at byte offset up256(4 * B*H*N_pad) (the layout include/fa.h states)."""
    npad = 128 * ((N + 127) // 128)
    off = (4 * B * H * npad + 255) // 256 * 256
    raw = ws[off:off + 4 * B * H * npad].view(torch.float32).view(B * H, npad)
    return raw.double().cpu().numpy(), npad


@pytest.mark.parametrize("B,N,H,d,dtype,causal", [
    (1, 300, 2, 64, "fp16", False),
    (2, 1000, 3, 128, "bf16", True),
    (4, 4096, 8, 128, "bf16", True),
])
def test_preprocess_d_matches_its_definition_and_the_oracle(B, N, H, d, dtype, causal):
    # D is computed by the preprocessing kernel from the forward's (rounded)
    # O and dO. Against rowsum(dO o O) of the same O in fp64, only fp32
    # accumulation error remains (a few ulps of sum |dO o O|). Against the
    # oracle's D (exact O), the gap is bounded by sum_k |dO_ik| * max|O_gpu -
    # O_exact|, which the forward's own O error gives.
    import exact_attention_119_b200 as fa
    from oracle import attention_forward
    case = Case(B, N, H, d, dtype, causal, seed=31)
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, case.scale, causal)
    ws = torch.zeros(fa.bwd_workspace_size(B, N, H, d, causal), dtype=torch.uint8, device="cuda")
    fa.backward(q, k, v, o, do, lse, case.scale, causal, workspace=ws)
    assert fa.check_device_status() == 0
    dd, npad = _workspace_d(ws, B, N, H)
    og = o.double().cpu().numpy()
    dof = case.f64["do"]
    prod = dof * og                                        # [B, N, H, d]
    want = prod.sum(axis=3).transpose(0, 2, 1).reshape(B * H, N)
    mag = np.abs(prod).sum(axis=3).transpose(0, 2, 1).reshape(B * H, N)
    got = dd[:, :N]
    assert np.all(np.abs(got - want) <= 1e-5 * mag + 1e-6)
    assert np.all(dd[:, N:] == 0.0)                        # pad rows
    # against the oracle (heads sampled at the large size)
    heads = [(0, 0), (B - 1, H - 1)] if N >= 4096 else None
    ro, _ = attention_forward(case.f64["q"], case.f64["k"], case.f64["v"], case.scale, causal)
    _, _, _, rd = attention_backward(case.f64["q"], case.f64["k"], case.f64["v"], dof, case.scale, causal,
                                     heads=heads)
    for b, h in heads or [(b, h) for b in range(B) for h in range(H)]:
        o_err = np.abs(og[b, :, h] - ro[b, :, h]).max()
        bound = np.abs(dof[b, :, h]).sum(axis=1) * o_err + 1e-5 * mag[b * H + h] + 1e-6
        assert np.all(np.abs(got[b * H + h] - rd[b, h]) <= bound), (b, h)

"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (a host process whose memory pool owns the whole device, code running
near capacity, loops that must not pay for the allocator). Its scratch is a
32 MiB array built into the library instead of a caller-provided workspace.

The test calls it through the C ABI twice in a row and compares each result
with fa_bwd's (which uses a caller-allocated workspace). Both run the same
deterministic kernels on the same inputs, so the results must be bitwise
equal; each is also within the gradient tolerance of the fp64 oracle. This
file is collected last on purpose; it also passes on its own in a fresh
process."""

import ctypes

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


@pytest.mark.parametrize("B,N,H,d,dtype,causal", [
    (2, 1000, 4, 128, "bf16", True),
    (2, 2048, 12, 64, "fp16", False),
])
def test_noalloc_matches_fa_bwd_twice(B, N, H, d, dtype, causal):
    import exact_attention_119_b200 as fa
    assert fa.bwd_workspace_size(B, N, H, d, causal) <= fa.noalloc_max_workspace()
    case = Case(B, N, H, d, dtype, causal, seed=21)
    q, k, v, do = (case.torch(n) for n in ("q", "k", "v", "do"))
    o, lse = fa.forward(q, k, v, case.scale, causal)
    ref = fa.backward(q, k, v, o, do, lse, case.scale, causal)
    heads = [(0, 0), (B - 1, H - 1)]
    exact = attention_backward(case.f64["q"], case.f64["k"], case.f64["v"], case.f64["do"], case.scale, causal,
                               heads=heads)[:3]
    for _ in range(2):
        got = fa.backward_noalloc(q, k, v, o, do, lse, case.scale, causal)
        assert fa.check_device_status() == 0
        for g, r, x in zip(got, ref, exact):
            assert torch.equal(g, r)
            gn = g.double().cpu().numpy()
            assert np.isfinite(gn).all()
            for b, h in heads:
                assert rel_fro(gn[b, :, h], x[b, :, h]) <= GRAD_REL_TOL


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # Rejected on the host before any launch, so tiny stand-in buffers are safe.
    import exact_attention_119_b200 as fa
    B, N, H, d = 1, 32768, 16, 128
    assert fa.bwd_workspace_size(B, N, H, d) > fa.noalloc_max_workspace()
    buf = torch.empty(64, dtype=torch.bfloat16, device="cuda")
    p = ctypes.c_void_p(buf.data_ptr())
    st = fa.library().fa_bwd_noalloc(p, p, p, p, p, p, p, p, p, B, N, H, d, 0.088, 0, 1, None)
    assert st == 5  # FA_ERR_WORKSPACE
    assert fa.check_device_status() == 0

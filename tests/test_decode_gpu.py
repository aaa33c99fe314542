"""Decode against a KV cache on a B200 (fa_decode through the C ABI) against
the fp64 oracle: O max-abs and LSE max-abs at the tolerances of the other
tests, ragged cache lengths, rows past each length filled with NaN (never
read), empty caches, causal and not, Nq = 1 .. 8."""

import numpy as np
import pytest

from exact_attention_119_b200 import inputs
from helpers import LSE_TOL, O_TOL, max_abs
from oracle import attention_forward_kvcache

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_attention_119_b200 as fa
    fa.library()


def make(B, Nq, H, d, Nmax, lens, dtype, seed):
    qb = inputs.make_tensor_bits((B, Nq, H, d), dtype, seed, 0)
    kb = inputs.make_tensor_bits((B, Nmax, H, d), dtype, seed, 1)
    vb = inputs.make_tensor_bits((B, Nmax, H, d), dtype, seed, 2)
    f = {n: inputs.bits_to_f64(b, dtype) for n, b in (("q", qb), ("k", kb), ("v", vb))}
    t = {n: inputs.bits_to_torch(b, dtype).cuda() for n, b in (("q", qb), ("k", kb), ("v", vb))}
    for b, L in enumerate(lens):  # rows past the length hold NaN: they must not reach the result
        t["k"][b, L:] = float("nan")
        t["v"][b, L:] = float("nan")
    return t, f, torch.tensor(lens, dtype=torch.int32, device="cuda")


def run_and_check(B, Nq, H, d, Nmax, lens, dtype, causal, seed):
    import exact_attention_119_b200 as fa
    t, f, cl = make(B, Nq, H, d, Nmax, lens, dtype, seed)
    scale = 1.0 / np.sqrt(d)
    o, lse = fa.decode(t["q"], t["k"], t["v"], cl, scale, causal)
    assert fa.check_device_status() == 0
    ro, rl = attention_forward_kvcache(f["q"], f["k"], f["v"], lens, scale, causal)
    og, lg = o.double().cpu().numpy(), lse.double().cpu().numpy()
    assert np.isfinite(og).all()
    assert max_abs(og, ro) <= O_TOL[dtype]
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(lg), fin)
    assert np.all(lg[~fin] == -np.inf)
    assert max_abs(lg[fin], rl[fin]) <= LSE_TOL if fin.any() else True


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Nq", [1, 3, 8])
@pytest.mark.parametrize("d,dtype", [(64, "fp16"), (128, "bf16"), (40, "fp16")])
def test_ragged_caches(d, dtype, Nq, causal):
    run_and_check(4, Nq, 3, d, 1000, [Nq, 64, 999, 513], dtype, causal, seed=Nq + d)


def test_empty_and_short_caches():
    # L = 0: no key (O = 0, LSE = -inf); causal rows before position 0 too.
    run_and_check(3, 4, 2, 64, 300, [0, 2, 300], "bf16", True, seed=3)


def test_long_cache_decoder_shape():
    # One new token of 8 sequences x 32 heads against 8192 cached positions
    # (d = 128, bf16): the serving shape the decode path is for.
    run_and_check(8, 1, 32, 128, 8192, [8192, 8000, 1, 4096, 8192, 77, 8191, 5000], "bf16", False, seed=7)


def test_matches_last_rows_of_causal_forward():
    # Decoding the last Nq positions of a cache equals those rows of the
    # causal forward over the whole sequence (each within the oracle bound).
    import exact_attention_119_b200 as fa
    B, N, H, d, Nq = 2, 700, 4, 128, 5
    qb, kb, vb = (inputs.make_tensor_bits((B, N, H, d), "bf16", 11, s) for s in range(3))
    q, k, v = (inputs.bits_to_torch(x, "bf16").cuda() for x in (qb, kb, vb))
    of, lf = fa.forward(q, k, v, None, True)
    od, ld = fa.decode(q[:, N - Nq:].contiguous(), k, v, torch.full((B,), N, dtype=torch.int32, device="cuda"),
                       None, True)
    assert fa.check_device_status() == 0
    assert (od.float() - of[:, N - Nq:].float()).abs().max().item() <= 2 * O_TOL["bf16"]
    assert (ld - lf[:, :, N - Nq:]).abs().max().item() <= 2 * LSE_TOL


def test_rejects_more_than_eight_rows():
    import exact_attention_119_b200 as fa
    q = torch.zeros(1, 9, 1, 64, dtype=torch.float16, device="cuda")
    kc = torch.zeros(1, 16, 1, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(fa.FAError):
        fa.decode(q, kc, kc, torch.tensor([16], dtype=torch.int32, device="cuda"))

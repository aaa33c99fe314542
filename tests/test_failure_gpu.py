"""Failure detection on a B200 without a GPU fault: a bounded device wait on a
flag that nothing sets gives up, the status word reports it, and the context
stays usable (the next attention call runs and is correct)."""

import math

import pytest

from helpers import O_TOL, Case, max_abs
from oracle import attention_forward

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


@pytest.mark.parametrize("which", [1, 2])
def test_bounded_wait_reports_timeout_and_context_survives(which):
    import exact_attention_119_b200 as fa
    assert fa.check_device_status() == 0
    fa.selftest_bounded_wait(which, limit_ms=50)
    assert fa.check_device_status() == 4          # FA_ERR_DEVICE_TIMEOUT
    assert fa.check_device_status() == 0          # read clears it
    case = Case(1, 300, 2, 64, "fp16", True, seed=11)
    o, _ = fa.forward(case.torch("q"), case.torch("k"), case.torch("v"), case.scale, True)
    assert fa.check_device_status() == 0
    ro, _ = attention_forward(case.f64["q"], case.f64["k"], case.f64["v"], case.scale, True)
    assert max_abs(o.double().cpu().numpy(), ro) <= O_TOL["fp16"]


def test_selftest_rejects_bad_arguments():
    import exact_attention_119_b200 as fa
    with pytest.raises(fa.FAError):
        fa.selftest_bounded_wait(3, 50)
    with pytest.raises(fa.FAError):
        fa.selftest_bounded_wait(1, 5000)

"""Pins of the oracle's dropout (CPU only): the Philox4x32-10 generator
against its published known-answer vectors, the mask's keep rate, the
unbiasedness of inverted dropout (the mean over masks is the undropped
result), p = 0 reducing to plain attention, and the gradients against central
finite differences with the mask held fixed."""

import json
import math
import os

import numpy as np
import pytest

from oracle import (attention_backward, attention_backward_dropout, attention_forward,
                    attention_forward_dropout, dropout_keep, dropout_threshold, philox4x32_10)

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_philox_known_answers():
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.json")) as f:
        kat = json.load(f)
    for vec in kat["vectors"]:
        c = [np.uint32(int(x, 16)) for x in vec["counter"]]
        k = [np.uint32(int(x, 16)) for x in vec["key"]]
        out = philox4x32_10(*c, *k)
        assert [int(x) for x in out] == [int(x, 16) for x in vec["output"]]


def test_threshold():
    assert dropout_threshold(0.0) == 0
    assert dropout_threshold(0.5) == 1 << 31
    assert dropout_threshold(0.25) == 1 << 30
    with pytest.raises(ValueError):
        dropout_threshold(1.0)


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
def test_keep_rate_and_independence(p):
    m = dropout_keep(1, 2, 4, 512, 512, p, seed=1234, offset=7)
    n = m.size
    keep = m.mean()
    sigma = math.sqrt(p * (1 - p) / n)
    assert abs(keep - (1 - p)) <= 5 * sigma
    # another head, offset or seed gives another mask; the same arguments the same one
    assert np.array_equal(m, dropout_keep(1, 2, 4, 512, 512, p, seed=1234, offset=7))
    for other in (dropout_keep(1, 3, 4, 512, 512, p, 1234, 7), dropout_keep(1, 2, 4, 512, 512, p, 1234, 8),
                  dropout_keep(1, 2, 4, 512, 512, p, 1235, 7)):
        agree = (other == m).mean()
        expect = p * p + (1 - p) * (1 - p)   # agreement rate of two independent masks
        assert abs(agree - expect) <= 5 * math.sqrt(expect * (1 - expect) / n)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_probability_is_plain_attention(causal):
    rng = np.random.default_rng(2)
    q, k, v, do = (rng.standard_normal((2, 9, 2, 4)) for _ in range(4))
    o, lse = attention_forward_dropout(q, k, v, 0.5, causal, 0.0, seed=3)
    ro, rl = attention_forward(q, k, v, 0.5, causal)
    np.testing.assert_allclose(o, ro, atol=1e-14)
    np.testing.assert_allclose(lse, rl, atol=1e-14)
    g = attention_backward_dropout(q, k, v, do, 0.5, causal, 0.0, seed=3)
    r = attention_backward(q, k, v, do, 0.5, causal)
    for a, b in zip(g, r):
        np.testing.assert_allclose(a, b, atol=1e-13)


def test_inverted_dropout_is_unbiased():
    # E[Z] = 1, so the mean of O over independent masks tends to the
    # undropped O, with the standard error of the mean.
    rng = np.random.default_rng(4)
    q, k, v = (rng.standard_normal((1, 6, 1, 3)) for _ in range(3))
    ro, _ = attention_forward(q, k, v, 0.6, False)
    p, n = 0.3, 3000
    outs = np.stack([attention_forward_dropout(q, k, v, 0.6, False, p, seed=s)[0] for s in range(n)])
    mean, se = outs.mean(axis=0), outs.std(axis=0) / math.sqrt(n)
    assert np.all(np.abs(mean - ro) <= 5 * se + 1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_dropout_gradients_match_finite_differences(causal):
    rng = np.random.default_rng(6)
    q, k, v, do = (rng.standard_normal((1, 7, 2, 3)) for _ in range(4))
    p, seed = 0.4, 99
    dq, dk, dv, dd = attention_backward_dropout(q, k, v, do, 0.7, causal, p, seed)

    def loss(qq, kk, vv):
        return float((attention_forward_dropout(qq, kk, vv, 0.7, causal, p, seed)[0] * do).sum())

    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        num = np.zeros_like(q)
        for idx in np.ndindex(*q.shape):
            args_p, args_m = [q.copy(), k.copy(), v.copy()], [q.copy(), k.copy(), v.copy()]
            args_p[which][idx] += h
            args_m[which][idx] -= h
            num[idx] = (loss(*args_p) - loss(*args_m)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)
    # D = rowsum(dO o O) holds with dropout too
    o, _ = attention_forward_dropout(q, k, v, 0.7, causal, p, seed)
    np.testing.assert_allclose(dd, (do * o).sum(axis=3).transpose(0, 2, 1), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_dropout_equals_fixed_length_batch(causal):
    # Equal-length sequences packed with cu_seqlens are the fixed-length batch,
    # dropout mask included (sequence b draws with b*H + h, i and j counted
    # from its first row).
    from oracle import attention_forward_varlen
    rng = np.random.default_rng(12)
    B, N, H, d = 3, 10, 2, 4
    q, k, v = (rng.standard_normal((B, N, H, d)) for _ in range(3))
    o, lse = attention_forward_dropout(q, k, v, 0.5, causal, 0.3, seed=77, offset=5)
    cu = np.arange(B + 1) * N
    ov, lv = attention_forward_varlen(q.reshape(B * N, H, d), k.reshape(B * N, H, d), v.reshape(B * N, H, d), cu,
                                      0.5, causal, dropout=(0.3, 77, 5))
    np.testing.assert_allclose(ov, o.reshape(B * N, H, d), atol=1e-13)
    np.testing.assert_allclose(lv, lse.transpose(1, 0, 2).reshape(H, B * N), atol=1e-13)

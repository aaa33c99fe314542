"""Pins of the oracle's variable-length and KV-cache functions (CPU only).

Each is tied to something other than itself: the fixed-length oracle (pinned
in test_oracle_pins.py) applied sequence by sequence, brute-force scalar loops
with math.fsum, independence of one sequence from another, central finite
differences, and the closed forms of degenerate cases.
"""

import math

import numpy as np
import pytest

from oracle import (attention_backward, attention_backward_varlen, attention_forward,
                    attention_forward_kvcache, attention_forward_varlen)

RNG = np.random.default_rng(4321)


def packed(total, H, d, scale=1.0):
    return RNG.standard_normal((total, H, d)) * scale


def brute_force_row(qrow, keys, vals, scale):
    """O and LSE of one query row by scalar loops (math.fsum)."""
    s = [scale * math.fsum(a * b for a, b in zip(qrow, kk)) for kk in keys]
    m = max(s)
    e = [math.exp(x - m) for x in s]
    z = math.fsum(e)
    o = [math.fsum(e[j] * vals[j][c] for j in range(len(keys))) / z for c in range(len(qrow))]
    return np.array(o), m + math.log(z)


LENS = [3, 0, 1, 7, 5]


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_equals_one_call_per_sequence(causal):
    cu = np.concatenate([[0], np.cumsum(LENS)])
    total, H, d = int(cu[-1]), 3, 4
    q, k, v, do = (packed(total, H, d) for _ in range(4))
    o, lse = attention_forward_varlen(q, k, v, cu, 0.6, causal)
    dq, dk, dv, dd = attention_backward_varlen(q, k, v, do, cu, 0.6, causal)
    for b, L in enumerate(LENS):
        a = int(cu[b])
        if L == 0:
            continue
        sl = slice(a, a + L)
        ro, rl = attention_forward(q[None, sl], k[None, sl], v[None, sl], 0.6, causal)
        np.testing.assert_allclose(o[sl], ro[0], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[:, sl], rl[0], rtol=0, atol=1e-13)
        g = attention_backward(q[None, sl], k[None, sl], v[None, sl], do[None, sl], 0.6, causal)
        for got, want in ((dq, g[0]), (dk, g[1]), (dv, g[2])):
            np.testing.assert_allclose(got[sl], want[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(dd[:, sl], g[3][0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_brute_force(causal):
    cu = np.concatenate([[0], np.cumsum(LENS)])
    total, H, d = int(cu[-1]), 2, 3
    q, k, v = (packed(total, H, d) for _ in range(3))
    o, lse = attention_forward_varlen(q, k, v, cu, 0.45, causal)
    for b, L in enumerate(LENS):
        a = int(cu[b])
        for i in range(L):
            last = i if causal else L - 1
            for h in range(H):
                ro, rl = brute_force_row(q[a + i, h], k[a:a + last + 1, h], v[a:a + last + 1, h], 0.45)
                np.testing.assert_allclose(o[a + i, h], ro, rtol=0, atol=1e-13)
                assert abs(lse[h, a + i] - rl) <= 1e-13


def test_varlen_sequences_do_not_see_each_other():
    # Changing every row of sequence 3 leaves the other sequences' outputs
    # and gradients unchanged.
    cu = np.concatenate([[0], np.cumsum(LENS)])
    total, H, d = int(cu[-1]), 2, 4
    q, k, v, do = (packed(total, H, d) for _ in range(4))
    o1, l1 = attention_forward_varlen(q, k, v, cu, 0.5, True)
    g1 = attention_backward_varlen(q, k, v, do, cu, 0.5, True)
    a, e = int(cu[3]), int(cu[4])
    for t in (q, k, v, do):
        t[a:e] = RNG.standard_normal((e - a, H, d)) * 5
    o2, l2 = attention_forward_varlen(q, k, v, cu, 0.5, True)
    g2 = attention_backward_varlen(q, k, v, do, cu, 0.5, True)
    keep = np.r_[0:a, e:total]
    np.testing.assert_array_equal(o1[keep], o2[keep])
    np.testing.assert_array_equal(l1[:, keep], l2[:, keep])
    for x, y in zip(g1[:3], g2[:3]):
        np.testing.assert_array_equal(x[keep], y[keep])
    assert not np.allclose(o1[a:e], o2[a:e])


@pytest.mark.parametrize("causal", [False, True])
def test_varlen_gradients_match_finite_differences(causal):
    lens = [3, 4]
    cu = np.concatenate([[0], np.cumsum(lens)])
    total, H, d = 7, 1, 3
    q, k, v, do = (packed(total, H, d) for _ in range(4))
    dq, dk, dv, _ = attention_backward_varlen(q, k, v, do, cu, 0.7, causal)

    def loss(qq, kk, vv):
        return float((attention_forward_varlen(qq, kk, vv, cu, 0.7, causal)[0] * do).sum())

    h = 1e-6
    for which, grad in ((0, dq), (1, dk), (2, dv)):
        args = [q, k, v]
        num = np.zeros_like(q)
        for idx in np.ndindex(*q.shape):
            plus = [a.copy() for a in args]
            minus = [a.copy() for a in args]
            plus[which][idx] += h
            minus[which][idx] -= h
            num[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        np.testing.assert_allclose(grad, num, rtol=1e-6, atol=1e-8)


def test_varlen_rejects_bad_offsets():
    q = packed(5, 1, 2)
    with pytest.raises(ValueError):
        attention_forward_varlen(q, q, q, [0, 3, 2, 5], 0.5)
    with pytest.raises(ValueError):
        attention_forward_varlen(q, q, q, [0, 3, 4], 0.5)


# ------------------------------------------------------------- KV-cache decode

@pytest.mark.parametrize("Nq", [1, 3])
def test_kvcache_causal_equals_last_rows_of_full_causal_attention(Nq):
    # A cache holding L positions, queried by its Nq newest ones, is the last
    # Nq rows of causal attention over all L positions.
    B, Nmax, H, d = 3, 11, 2, 4
    lens = [Nq, 6, 11]
    Q, K, V = (RNG.standard_normal((B, Nmax, H, d)) for _ in range(3))
    q = np.stack([Q[b, lens[b] - Nq:lens[b]] for b in range(B)])
    o, lse = attention_forward_kvcache(q, K, V, lens, 0.4, causal=True)
    for b, L in enumerate(lens):
        ro, rl = attention_forward(Q[None, b, :L], K[None, b, :L], V[None, b, :L], 0.4, True)
        np.testing.assert_allclose(o[b], ro[0, L - Nq:], rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[b], rl[0][:, L - Nq:], rtol=0, atol=1e-13)


def test_kvcache_noncausal_brute_force_and_ignores_rows_past_the_length():
    B, Nmax, H, d, Nq = 2, 9, 2, 3, 2
    lens = [4, 9]
    q = RNG.standard_normal((B, Nq, H, d))
    K, V = (RNG.standard_normal((B, Nmax, H, d)) for _ in range(2))
    o, lse = attention_forward_kvcache(q, K, V, lens, 0.8, causal=False)
    K2, V2 = K.copy(), V.copy()
    K2[0, 4:] = np.nan       # rows past the cache length are never read
    V2[0, 4:] = np.inf
    o2, lse2 = attention_forward_kvcache(q, K2, V2, lens, 0.8, causal=False)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)
    for b, L in enumerate(lens):
        for t in range(Nq):
            for h in range(H):
                ro, rl = brute_force_row(q[b, t, h], K[b, :L, h], V[b, :L, h], 0.8)
                np.testing.assert_allclose(o[b, t, h], ro, rtol=0, atol=1e-13)
                assert abs(lse[b, h, t] - rl) <= 1e-13


def test_kvcache_degenerate_cases():
    q = RNG.standard_normal((2, 1, 1, 3))
    K, V = RNG.standard_normal((2, 4, 1, 3)), RNG.standard_normal((2, 4, 1, 3))
    o, lse = attention_forward_kvcache(q, K, V, [1, 0], 0.5)
    np.testing.assert_allclose(o[0, 0, 0], V[0, 0, 0], atol=1e-15)     # one key: its value
    assert abs(lse[0, 0, 0] - 0.5 * float(q[0, 0, 0] @ K[0, 0, 0])) <= 1e-14
    assert np.all(o[1] == 0.0) and np.all(np.isneginf(lse[1]))        # empty cache


# ----------------------------------------------------------- planted mistakes
# Copies of the new oracle functions with one slip each (written here, on the
# CPU); the pins above must catch every one.

def _varlen_mutant(kind):
    def fwd(q, k, v, cu, scale, causal):
        total, H, d = q.shape
        o = np.zeros_like(q)
        bounds = [(0, total)] if kind == "no_boundaries" else list(zip(cu[:-1], cu[1:]))
        for a, e in bounds:
            if kind == "drop_last_row":
                e = max(a, e - 1)
            if e == a:
                continue
            for h in range(H):
                s = scale * q[a:e, h] @ k[a:e, h].T
                if causal:
                    s[np.triu_indices(e - a, 1)] = -np.inf
                p = np.exp(s - s.max(axis=1, keepdims=True))
                o[a:e, h] = (p / p.sum(axis=1, keepdims=True)) @ v[a:e, h]
        return o
    return fwd


@pytest.mark.parametrize("kind", ["no_boundaries", "drop_last_row"])
def test_pins_catch_varlen_slips(kind):
    cu = np.concatenate([[0], np.cumsum(LENS)])
    rng = np.random.default_rng(8)
    q, k, v = (rng.standard_normal((int(cu[-1]), 2, 3)) for _ in range(3))
    o = _varlen_mutant(kind)(q, k, v, cu, 0.6, True)
    caught = False
    for b, L in enumerate(LENS):
        a = int(cu[b])
        if L:
            ro, _ = attention_forward(q[None, a:a + L], k[None, a:a + L], v[None, a:a + L], 0.6, True)
            caught |= not np.allclose(o[a:a + L], ro[0], atol=1e-9)
    assert caught


def _kvcache_mutant(kind):
    def fwd(q, kc, vc, lens, scale, causal):
        B, Nq, H, d = q.shape
        o = np.zeros_like(q)
        for b in range(B):
            L = kc.shape[1] if kind == "whole_cache" else lens[b]
            for t in range(Nq):
                last = (t if kind == "top_left" else L - Nq + t) if causal else L - 1
                for h in range(H):
                    s = scale * kc[b, :last + 1, h] @ q[b, t, h]
                    e = np.exp(s - s.max())
                    o[b, t, h] = e @ vc[b, :last + 1, h] / e.sum()
        return o
    return fwd


@pytest.mark.parametrize("kind", ["top_left", "whole_cache"])
def test_pins_catch_kvcache_slips(kind):
    rng = np.random.default_rng(9)
    B, Nmax, H, d, Nq = 2, 8, 1, 3, 3
    lens = [5, 8]
    Q, K, V = (rng.standard_normal((B, Nmax, H, d)) for _ in range(3))
    q = np.stack([Q[b, lens[b] - Nq:lens[b]] for b in range(B)])
    o = _kvcache_mutant(kind)(q, K, V, lens, 0.4, True)
    ro, _ = attention_forward(Q[None, 0, :5], K[None, 0, :5], V[None, 0, :5], 0.4, True)
    assert not np.allclose(o[0], ro[0, 5 - Nq:], atol=1e-9)

"""Pins of the fp64 oracle to things other than itself (CPU only).

Each pin is chosen so that a plausible slip in the oracle (a dropped scale, a
transposed operand, softmax over the wrong axis, the causal mask on the wrong
side of the diagonal, a wrong sign in dS) fails at least one of them; the
mutation tests at the end plant such slips in copies of the oracle and check
that the pins catch them.
"""

import json
import math
import os
import re
from fractions import Fraction

import numpy as np
import pytest

from oracle import attention_backward, attention_forward, default_scale, online_softmax_forward

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def rand(*shape, scale=1.0, rng=None):
    return (rng or RNG).standard_normal(shape) * scale


# ----------------------------------------------------------------- forward pins

@pytest.mark.parametrize("causal", [False, True])
def test_rows_of_p_sum_to_one(causal):
    # With V = identity (d = N), O = P exactly: its rows are the softmax rows.
    N = 9
    q, k = rand(1, N, 1, N), rand(1, N, 1, N)
    v = np.eye(N).reshape(1, N, 1, N)
    p, _ = attention_forward(q, k, v, 0.7, causal)
    p = p[0, :, 0, :]
    assert np.all(p >= 0)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, atol=1e-12)
    if causal:
        assert np.all(p[np.triu_indices(N, 1)] == 0.0)   # keys after the query get nothing
        assert np.all(p[np.tril_indices(N)] > 0.0)


@pytest.mark.parametrize("causal", [False, True])
def test_constant_v_returns_v(causal):
    B, N, H, d = 2, 13, 3, 5
    q, k = rand(B, N, H, d, scale=3.0), rand(B, N, H, d, scale=3.0)
    row = rand(d)
    v = np.broadcast_to(row, (B, N, H, d)).copy()
    o, _ = attention_forward(q, k, v, 0.3, causal)
    np.testing.assert_allclose(o, v, atol=1e-12)


def test_single_key_returns_its_value():
    q, k, v = rand(2, 1, 3, 4), rand(2, 1, 3, 4), rand(2, 1, 3, 4)
    s = 0.37
    for causal in (False, True):
        o, lse = attention_forward(q, k, v, s, causal)
        np.testing.assert_allclose(o, v, atol=1e-14)
        np.testing.assert_allclose(lse, s * np.einsum("bnhd,bnhd->bhn", q, k), atol=1e-14)


def test_causal_row0_is_v0():
    B, N, H, d = 2, 11, 2, 6
    q, k, v = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    s = default_scale(d)
    o, lse = attention_forward(q, k, v, s, True)
    np.testing.assert_allclose(o[:, 0], v[:, 0], atol=1e-14)
    np.testing.assert_allclose(lse[:, :, 0], s * np.einsum("bhd,bhd->bh", q[:, 0], k[:, 0]), atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_zero_queries_give_uniform_weights(causal):
    B, N, H, d = 1, 10, 2, 3
    q = np.zeros((B, N, H, d))
    k, v = rand(B, N, H, d), rand(B, N, H, d)
    o, lse = attention_forward(q, k, v, 0.5, causal)
    for i in range(N):
        cnt = i + 1 if causal else N
        np.testing.assert_allclose(o[:, i], v[:, :cnt].mean(axis=1), atol=1e-13)
        np.testing.assert_allclose(lse[:, :, i], math.log(cnt), atol=1e-13)


@pytest.mark.parametrize("causal", [False, True])
def test_key_shift_invariance(causal):
    B, N, H, d = 1, 12, 2, 4
    q, k, v = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    w = rand(1, 1, H, d)
    s = 0.8
    o1, l1 = attention_forward(q, k, v, s, causal)
    o2, l2 = attention_forward(q, k + w, v, s, causal)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    shift = s * np.einsum("bnhd,hd->bhn", q, w[0, 0])
    np.testing.assert_allclose(l2, l1 + shift, atol=1e-12)


def test_key_value_permutation_invariance():
    B, N, H, d = 2, 15, 2, 4
    q, k, v = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    perm = RNG.permutation(N)
    o1, l1 = attention_forward(q, k, v, 0.6, False)
    o2, l2 = attention_forward(q, k[:, perm], v[:, perm], 0.6, False)
    np.testing.assert_allclose(o2, o1, atol=1e-12)
    np.testing.assert_allclose(l2, l1, atol=1e-12)


def brute_force(q, k, v, scale, causal):
    """Independent scalar triple loop with exactly rounded sums (math.fsum)."""
    B, N, H, d = q.shape
    o = np.zeros((B, N, H, d))
    lse = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            for i in range(N):
                logits = []
                for j in range(N):
                    if causal and j > i:
                        continue
                    logits.append((j, scale * math.fsum(q[b, i, h, t] * k[b, j, h, t] for t in range(d))))
                mx = max(x for _, x in logits)
                w = [(j, math.exp(x - mx)) for j, x in logits]
                z = math.fsum(e for _, e in w)
                lse[b, h, i] = mx + math.log(z)
                for t in range(d):
                    o[b, i, h, t] = math.fsum(e * v[b, j, h, t] for j, e in w) / z
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(1, 1), (3, 2), (8, 4), (7, 3)])
def test_brute_force_tiny(N, d, causal):
    rng = np.random.default_rng(N * 10 + d)
    q, k, v = (rng.standard_normal((2, N, 2, d)) * 2 for _ in range(3))
    o, lse = attention_forward(q, k, v, 0.9, causal)
    ob, lb = brute_force(q, k, v, 0.9, causal)
    np.testing.assert_allclose(o, ob, atol=1e-13)
    np.testing.assert_allclose(lse, lb, atol=1e-13)


def test_row_sampling_matches_full():
    B, N, H, d = 1, 40, 2, 8
    q, k, v = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    rows = np.array([0, 1, 17, 39])
    for causal in (False, True):
        of, lf = attention_forward(q, k, v, 0.4, causal)
        os_, ls = attention_forward(q, k, v, 0.4, causal, rows=rows)
        np.testing.assert_array_equal(os_[:, rows], of[:, rows])
        np.testing.assert_array_equal(ls[:, :, rows], lf[:, :, rows])
        assert np.isnan(os_[:, 2]).all()


def test_row_blocking_matches_unblocked(monkeypatch):
    import oracle.attention as oa
    B, N, H, d = 1, 50, 1, 4
    q, k, v = rand(B, N, H, d), rand(B, N, H, d), rand(B, N, H, d)
    o1, l1 = attention_forward(q, k, v, 0.5, True)
    monkeypatch.setattr(oa, "ROW_BLOCK", 7)
    o2, l2 = oa.attention_forward(q, k, v, 0.5, True)
    np.testing.assert_allclose(o2, o1, atol=1e-14)
    np.testing.assert_allclose(l2, l1, atol=1e-14)


@pytest.mark.parametrize("causal", [False, True])
def test_online_recurrence_equals_direct(causal):
    # [P3] §3.2: the tiled recurrence reaches the global softmax exactly.
    B, N, H, d = 1, 37, 2, 6
    q, k, v = rand(B, N, H, d, scale=2.0), rand(B, N, H, d, scale=2.0), rand(B, N, H, d)
    o, lse = attention_forward(q, k, v, 0.7, causal)
    rng = np.random.default_rng(7)
    for _ in range(5):
        cuts = sorted(rng.choice(np.arange(1, N), size=rng.integers(1, 8), replace=False))
        sizes = list(np.diff([0, *cuts, N]))
        ot, lt = online_softmax_forward(q, k, v, 0.7, causal, sizes)
        np.testing.assert_allclose(ot, o, atol=1e-12)
        np.testing.assert_allclose(lt, lse, atol=1e-12)


# ----------------------------------------------------------- hand-worked example

def _ev(expr):
    m = re.fullmatch(r"(?:(-?\d+(?:/\d+)?)\*)?ln\((\d+(?:/\d+)?)\)", expr)
    if m:
        c = Fraction(m.group(1)) if m.group(1) else Fraction(1)
        return float(c) * math.log(float(Fraction(m.group(2))))
    return float(Fraction(expr))


def _hand_case():
    with open(os.path.join(GOLDEN, "hand_2x2.json")) as f:
        g = json.load(f)
    inp = g["inputs"]
    # embed the case at (b=1, h=2) of a larger random batch to pin the indexing
    B, N, H, d = 2, 2, 3, 1
    q, k, v, do = (RNG.standard_normal((B, N, H, d)) for _ in range(4))
    for arr, key in ((q, "q"), (k, "k"), (v, "v"), (do, "do")):
        arr[1, :, 2, 0] = inp[key]
    return g, _ev(inp["scale"]), q, k, v, do


@pytest.mark.parametrize("mode", ["noncausal", "causal"])
def test_hand_worked_example(mode):
    g, scale, q, k, v, do = _hand_case()
    causal = mode == "causal"
    exp = {key: np.array([_ev(x) for x in vals]) for key, vals in g[mode].items()}
    o, lse = attention_forward(q, k, v, scale, causal)
    dq, dk, dv, dd = attention_backward(q, k, v, do, scale, causal)
    np.testing.assert_allclose(o[1, :, 2, 0], exp["o"], atol=1e-13)
    np.testing.assert_allclose(lse[1, 2, :], exp["lse"], atol=1e-13)
    np.testing.assert_allclose(dq[1, :, 2, 0], exp["dq"], atol=1e-13)
    np.testing.assert_allclose(dk[1, :, 2, 0], exp["dk"], atol=1e-13)
    np.testing.assert_allclose(dv[1, :, 2, 0], exp["dv"], atol=1e-13)
    np.testing.assert_allclose(dd[1, 2, :], exp["D"], atol=1e-13)


# ---------------------------------------------------------------- gradient pins

def loss(q, k, v, do, scale, causal):
    o, _ = attention_forward(q, k, v, scale, causal)
    return float(np.sum(do * o))


def fd_grads(q, k, v, do, scale, causal, h=1e-6):
    grads = []
    for which in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(args[which])
        it = np.nditer(args[which], flags=["multi_index"])
        for _ in it:
            idx = it.multi_index
            x0 = args[which][idx]
            args[which][idx] = x0 + h
            lp = loss(*args, do, scale, causal)
            args[which][idx] = x0 - h
            lm = loss(*args, do, scale, causal)
            args[which][idx] = x0
            g[idx] = (lp - lm) / (2 * h)
        grads.append(g)
    return grads


def rel(a, b):
    return np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("N,d", [(5, 3), (16, 8)])
def test_gradients_match_finite_differences(N, d, causal):
    rng = np.random.default_rng(N + d + causal)
    q, k, v, do = (rng.standard_normal((1, N, 2, d)) for _ in range(4))
    s = default_scale(d)
    dq, dk, dv, _ = attention_backward(q, k, v, do, s, causal)
    fq, fk, fv = fd_grads(q, k, v, do, s, causal)
    assert rel(dq, fq) < 1e-6
    assert rel(dk, fk) < 1e-6
    assert rel(dv, fv) < 1e-6


@pytest.mark.parametrize("causal", [False, True])
def test_gradient_invariants(causal):
    B, N, H, d = 2, 21, 2, 5
    q, k, v, do = (rand(B, N, H, d) for _ in range(4))
    s = 0.45
    o, _ = attention_forward(q, k, v, s, causal)
    dq, dk, dv, dd = attention_backward(q, k, v, do, s, causal)
    # rows of P sum to 1  =>  sum_j dV_j = sum_i dO_i
    np.testing.assert_allclose(dv.sum(axis=1), do.sum(axis=1), atol=1e-12)
    # rows of dS sum to 0  =>  sum_j dK_j = 0
    np.testing.assert_allclose(dk.sum(axis=1), 0.0, atol=1e-12)
    # D = rowsum(P o dP) = rowsum(dO o O)
    np.testing.assert_allclose(dd, np.einsum("bnhd,bnhd->bhn", do, o), rtol=1e-12, atol=1e-12)


def test_head_sampling_matches_full():
    B, N, H, d = 2, 9, 3, 4
    q, k, v, do = (rand(B, N, H, d) for _ in range(4))
    full = attention_backward(q, k, v, do, 0.5, True)
    part = attention_backward(q, k, v, do, 0.5, True, heads=[(1, 2)])
    for f, p in zip(full, part):
        np.testing.assert_array_equal(p[1, :, 2] if f.ndim == 4 else p[1, 2], f[1, :, 2] if f.ndim == 4 else f[1, 2])


# ----------------------------------------------------------- planted mistakes
# Copies of the oracle with one slip each, run through the pins above; each
# slip must be caught. The slips are planted here, on the CPU, never on a GPU.

def _fwd_mutant(kind):
    def fwd(q, k, v, scale, causal):
        B, N, H, d = q.shape
        o = np.zeros_like(q)
        lse = np.zeros((B, H, N))
        for b in range(B):
            for h in range(H):
                s = (1.0 if kind == "no_scale" else scale) * q[b, :, h] @ k[b, :, h].T
                if causal:
                    tri = np.tril_indices(N, -1) if kind == "mask_flipped" else np.triu_indices(N, 1)
                    s[tri] = -np.inf
                ax = 0 if kind == "softmax_axis" else 1
                m = s.max(axis=ax, keepdims=True)
                e = np.exp(s - m)
                p = e / e.sum(axis=ax, keepdims=True)
                o[b, :, h] = (p.T if kind == "p_transposed" else p) @ v[b, :, h]
                lse[b, h] = np.log(np.exp(s).sum(axis=1))
        return o, lse
    return fwd


@pytest.mark.parametrize("kind", ["no_scale", "mask_flipped", "softmax_axis", "p_transposed"])
def test_pins_catch_forward_slips(kind):
    fwd = _fwd_mutant(kind)
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((1, 6, 1, 3)) * 2 for _ in range(3))
    causal = kind == "mask_flipped"
    o, _ = fwd(q, k, v, 0.7, causal)
    ob, _ = brute_force(q, k, v, 0.7, causal)
    assert not np.allclose(o, ob, atol=1e-6)


def _bwd_mutant(kind):
    def bwd(q, k, v, do, scale, causal):
        B, N, H, d = q.shape
        dq, dk, dv = (np.zeros_like(q) for _ in range(3))
        for b in range(B):
            for h in range(H):
                qh, kh, vh, doh = q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h]
                s = scale * qh @ kh.T
                if causal:
                    s[np.triu_indices(N, 1)] = -np.inf
                e = np.exp(s - s.max(axis=1, keepdims=True))
                p = e / e.sum(axis=1, keepdims=True)
                dvh = (p if kind == "dv_no_transpose" else p.T) @ doh
                dp = doh @ vh.T
                D = (p * dp).sum(axis=1)
                ds = p * (dp + D[:, None]) if kind == "ds_sign" else p * (dp - D[:, None])
                dq[b, :, h] = (1.0 if kind == "dq_no_scale" else scale) * ds @ kh
                dk[b, :, h] = scale * (ds if kind == "dk_no_transpose" else ds.T) @ qh
                dv[b, :, h] = dvh
        return dq, dk, dv
    return bwd


@pytest.mark.parametrize("kind", ["dv_no_transpose", "ds_sign", "dq_no_scale", "dk_no_transpose"])
def test_pins_catch_backward_slips(kind):
    bwd = _bwd_mutant(kind)
    rng = np.random.default_rng(5)
    q, k, v, do = (rng.standard_normal((1, 5, 1, 3)) for _ in range(4))
    s = default_scale(3)
    g = bwd(q, k, v, do, s, False)
    f = fd_grads(q, k, v, do, s, False)
    assert max(rel(a, b) for a, b in zip(g, f)) > 1e-3

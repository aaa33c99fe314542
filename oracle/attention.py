"""fp64 CPU oracle for exact scaled-dot-product attention, forward and backward.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The product path
(``exact_attention_119_b200``) never imports it and shares no code with it.

Sources (the web pages this build follows; cited by title and section):

* [P3] "从Attention矩阵到显存读写：FlashAttention真正解决的痛点" (lab write-up,
  dpshk.com): §2.1 the three-step definition S = Q K^T, P = softmax(S) along
  the last dimension, O = P V; §3.2 the online-softmax recurrence with running
  row max m and exp-sum l; §3.3 recomputation in the backward pass; §4.2 the
  [batch, seqlen, heads, head_dim] layout, ``softmax_scale`` (default 1/sqrt(d))
  and ``causal``.
* [P4] "使用FlashAttention优化PyTorch模型注意力计算" (tiemojia.cn), section
  "FlashAttention 是如何做到又快又省内存的": the einsum form of standard
  attention, scores divided by sqrt(d_head), softmax over the key axis.

The method is mathematically the plain definition ([P3] §3.2 states the tiled
form is equivalent to the global softmax; [P4] calls it "数学上等价"), so the
forward oracle *is* that definition, materialising S and P in full for each
(batch, head). The pages give no backward formulas; the backward oracle is the
textbook chain rule through the softmax Jacobian (the plain reading):

    dV = P^T dO;  dP = dO V^T;  D_i = sum_j P_ij dP_ij;  dS = P o (dP - D)
    dQ = scale * dS K;  dK = scale * dS^T Q

``online_softmax_forward`` restates the tiled recurrence of [P3] §3.2 step by
step (in fp64); it is pinned against the direct definition in the tests.

Masking reading: ``causal`` keeps key j for query i iff j <= i (queries and keys
have the same length, so the mask is aligned top-left). Row logsumexp (LSE) is
the natural log of sum_j exp(scale * q_i . k_j) over kept keys; the pages do not
define it, it is what the backward recompute needs.

Every function here is pinned by a test in ``tests/test_oracle_pins.py`` to
something other than itself (closed forms, invariants, brute force, a hand-worked
example, central finite differences).
"""

from __future__ import annotations

import math

import numpy as np

ROW_BLOCK = 512  # rows of S materialised at once for long sequences


def _as_f64(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float64)
    if a.ndim != 4:
        raise ValueError("expected a [batch, seqlen, heads, head_dim] array")
    return a


def _scores(qh: np.ndarray, kh: np.ndarray, scale: float, rows: np.ndarray, causal: bool) -> np.ndarray:
    """S = scale * Q K^T for the given query rows of one head ([P3] §2.1 step 1).

    Causal: entries with key index j > query index i are -inf (excluded).
    """
    s = scale * (qh[rows] @ kh.T)
    if causal:
        keys = np.arange(kh.shape[0])
        s[keys[None, :] > rows[:, None]] = -np.inf
    return s


def _softmax_rows(s: np.ndarray):
    """P = softmax(S) along the key axis ([P3] §2.1 step 2), and the row LSE."""
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    l = e.sum(axis=1, keepdims=True)
    return e / l, (m + np.log(l))[:, 0]


def attention_forward(q, k, v, scale: float, causal: bool = False, rows=None):
    """O = softmax(scale Q K^T [+causal mask]) V and LSE, in fp64.

    q, k, v: [B, N, H, d]. Returns (O [B, N, H, d], LSE [B, H, N]).
    ``rows``: optional 1-D array of query rows to evaluate (each row is
    independent); the other rows of O / LSE are NaN.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, N, H, d = q.shape
    if k.shape != (B, N, H, d) or v.shape != (B, N, H, d):
        raise ValueError("q, k, v must share the shape [B, N, H, d]")
    all_rows = np.arange(N) if rows is None else np.asarray(rows, dtype=np.int64)
    o = np.full((B, N, H, d), np.nan)
    lse = np.full((B, H, N), np.nan)
    for b in range(B):
        for h in range(H):
            qh, kh, vh = q[b, :, h, :], k[b, :, h, :], v[b, :, h, :]
            for r0 in range(0, len(all_rows), ROW_BLOCK):
                rr = all_rows[r0:r0 + ROW_BLOCK]
                p, lse_rows = _softmax_rows(_scores(qh, kh, scale, rr, causal))
                o[b, rr, h, :] = p @ vh          # [P3] §2.1 step 3
                lse[b, h, rr] = lse_rows
    return o, lse


def _head_backward(qh, kh, vh, doh, scale: float, causal: bool):
    """dQ, dK, dV and D of one head (textbook chain rule through softmax)."""
    rows = np.arange(qh.shape[0])
    p, _ = _softmax_rows(_scores(qh, kh, scale, rows, causal))
    dvh = p.T @ doh
    dp = doh @ vh.T
    drow = (p * dp).sum(axis=1)
    ds = p * (dp - drow[:, None])
    return scale * (ds @ kh), scale * (ds.T @ qh), dvh, drow


def attention_backward(q, k, v, do, scale: float, causal: bool = False, heads=None):
    """Gradients (dQ, dK, dV) of L = sum(dO o O) for the attention above, fp64.

    ``heads``: optional list of (b, h) pairs to evaluate (dK/dV of a head need
    every query row, so sampling is per head); other heads are NaN.
    Also returns D [B, H, N] = rowsum(P o dP), which equals rowsum(dO o O).
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, N, H, d = q.shape
    dq = np.full_like(q, np.nan)
    dk = np.full_like(q, np.nan)
    dv = np.full_like(q, np.nan)
    dd = np.full((B, H, N), np.nan)
    pairs = [(b, h) for b in range(B) for h in range(H)] if heads is None else list(heads)
    for b, h in pairs:
        dq[b, :, h, :], dk[b, :, h, :], dv[b, :, h, :], dd[b, h, :] = _head_backward(
            q[b, :, h, :], k[b, :, h, :], v[b, :, h, :], do[b, :, h, :], scale, causal)
    return dq, dk, dv, dd


def online_softmax_forward(q, k, v, scale: float, causal: bool, tile_sizes):
    """The tiled online-softmax forward of [P3] §3.2, one key tile at a time.

    For each query row, keep the running max m and exp-sum l; for each key tile
    j with local scores s: m_new = max(m, max(s)); O <- O * e^(m - m_new) +
    e^(s - m_new) V_j; l <- l * e^(m - m_new) + sum e^(s - m_new); at the end
    O <- O / l. ``tile_sizes`` lists the widths of the consecutive key tiles
    (they must add up to N). Returns (O, LSE) with LSE = m + ln l.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, N, H, d = q.shape
    if sum(tile_sizes) != N:
        raise ValueError("tile sizes must cover the key axis exactly")
    o = np.empty((B, N, H, d))
    lse = np.empty((B, H, N))
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            qh, kh, vh = q[b, :, h, :], k[b, :, h, :], v[b, :, h, :]
            m = np.full(N, -np.inf)
            l = np.zeros(N)
            acc = np.zeros((N, d))
            start = 0
            for width in tile_sizes:
                cols = np.arange(start, start + width)
                s = scale * (qh @ kh[cols].T)
                if causal:
                    s[cols[None, :] > rows[:, None]] = -np.inf
                m_new = np.maximum(m, s.max(axis=1))
                # rows with nothing kept so far keep m = -inf; guard their factors
                alive = np.isfinite(m_new)
                alpha = np.where(alive, np.exp(np.where(alive, m - m_new, 0.0)), 1.0)
                e = np.where(alive[:, None], np.exp(s - np.where(alive, m_new, 0.0)[:, None]), 0.0)
                acc = acc * alpha[:, None] + e @ vh[cols]
                l = l * alpha + e.sum(axis=1)
                m = m_new
                start += width
            o[b, :, h, :] = acc / l[:, None]
            lse[b, h, :] = m + np.log(l)
    return o, lse


def default_scale(d: int) -> float:
    """softmax_scale=None means 1/sqrt(head_dim) ([P3] §4.2 and §6.2)."""
    return 1.0 / math.sqrt(d)


# ------------------------------------------------------------ variable length

def _as_packed(x) -> np.ndarray:
    a = np.asarray(x, dtype=np.float64)
    if a.ndim != 3:
        raise ValueError("expected a packed [total, heads, head_dim] array")
    return a


def _seq_bounds(cu_seqlens, total: int):
    cu = [int(c) for c in cu_seqlens]
    if cu[0] != 0 or cu[-1] != total or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must start at 0, not decrease and end at total")
    return list(zip(cu[:-1], cu[1:]))


def attention_forward_varlen(q, k, v, cu_seqlens, scale: float, causal: bool = False, dropout=None):
    """Variable-length batch, packed without padding ([P3] §4.2, third pitfall:
    variable-length sequences go through flash_attn_varlen_func).

    q, k, v: [total, H, d]; sequence b owns rows cu_seqlens[b] ..
    cu_seqlens[b+1] - 1 of all three and attends only to itself (causal: key
    j of the sequence for query i of the sequence iff j <= i). Each sequence is
    the plain definition on its own rows. Returns O [total, H, d] and
    LSE [H, total] (row r of the packed tensors at column r). ``dropout``:
    optional (p, seed, offset), the mask of dropout_keep() with b the
    sequence's index and i, j counted from its first row.
    """
    q, k, v = _as_packed(q), _as_packed(k), _as_packed(v)
    total, H, d = q.shape
    o = np.full((total, H, d), np.nan)
    lse = np.full((H, total), np.nan)
    bounds = _seq_bounds(cu_seqlens, total)
    seq_index = {ae: b for b, ae in enumerate(bounds)}
    for a, e in bounds:
        if e == a:
            continue
        rows = np.arange(e - a)
        for h in range(H):
            p, lse_rows = _softmax_rows(_scores(q[a:e, h], k[a:e, h], scale, rows, causal))
            if dropout is not None:
                pd, seed, offset = dropout
                p = p * dropout_keep(seq_index[a, e], h, H, e - a, e - a, pd, seed, offset) / (1.0 - pd)
            o[a:e, h] = p @ v[a:e, h]
            lse[h, a:e] = lse_rows
    return o, lse


def attention_backward_varlen(q, k, v, do, cu_seqlens, scale: float, causal: bool = False):
    """Gradients of the variable-length forward above: each sequence's dQ, dK,
    dV and D by the chain rule on its own rows. Returns dQ, dK, dV
    [total, H, d] and D [H, total]."""
    q, k, v, do = _as_packed(q), _as_packed(k), _as_packed(v), _as_packed(do)
    total, H, d = q.shape
    dq, dk, dv = (np.full((total, H, d), np.nan) for _ in range(3))
    dd = np.full((H, total), np.nan)
    for a, e in _seq_bounds(cu_seqlens, total):
        if e == a:
            continue
        for h in range(H):
            dq[a:e, h], dk[a:e, h], dv[a:e, h], dd[h, a:e] = _head_backward(
                q[a:e, h], k[a:e, h], v[a:e, h], do[a:e, h], scale, causal)
    return dq, dk, dv, dd


# ----------------------------------------------------------- KV-cache decode

def attention_forward_kvcache(q, k_cache, v_cache, cache_seqlens, scale: float, causal: bool = False):
    """Decode step against a key/value cache ([P3] §6.1: inference with a KV
    cache whose length grows one step at a time).

    q: [B, Nq, H, d], the Nq newest positions of each sequence; k_cache,
    v_cache: [B, Nmax, H, d], of which batch b holds L_b = cache_seqlens[b]
    valid rows (the Nq newest included). Query t of batch b sits at position
    L_b - Nq + t; it attends keys 0 .. L_b - 1, or with ``causal`` keys
    0 .. L_b - Nq + t (its own position and earlier). A query with no key to
    attend (L_b - Nq + t < 0 under ``causal``, or L_b = 0) gets O = 0 and
    LSE = -inf. Returns O [B, Nq, H, d] and LSE [B, H, Nq].
    """
    q, kc, vc = _as_f64(q), _as_f64(k_cache), _as_f64(v_cache)
    B, Nq, H, d = q.shape
    o = np.zeros((B, Nq, H, d))
    lse = np.full((B, H, Nq), -np.inf)
    for b in range(B):
        L = int(cache_seqlens[b])
        if not 0 <= L <= kc.shape[1]:
            raise ValueError("cache length out of range")
        for t in range(Nq):
            last = L - 1 if not causal else L - Nq + t
            if last < 0:
                continue
            for h in range(H):
                s = scale * (kc[b, :last + 1, h] @ q[b, t, h])
                m = s.max()
                e = np.exp(s - m)
                o[b, t, h] = (e @ vc[b, :last + 1, h]) / e.sum()
                lse[b, h, t] = m + np.log(e.sum())
    return o, lse


# ------------------------------------------------------------------ dropout

def dropout_threshold(p: float) -> int:
    """The integer form of a dropout probability: an element is dropped when
    its 32-bit random word is below floor(p * 2^32) (so p = 0 drops nothing).
    Both sides receive this integer; no floating point decides a mask bit."""
    if not 0.0 <= p < 1.0:
        raise ValueError("dropout probability must be in [0, 1)")
    return min(int(p * 4294967296.0), 4294967295)


def dropout_keep(b: int, h: int, H: int, nq: int, nk: int, p: float, seed: int, offset: int) -> np.ndarray:
    """Keep mask [nq, nk] of head (b, h) (b: the sequence when variable-length).

    The dropout of P ([P2] usage line and [P3] §4.2: flash_attn_func takes
    dropout_p) needs a mask that the backward pass can regenerate instead of
    storing; the pages give no generator, so this one is Philox4x32-10 (see
    oracle/philox.py) with key (seed mod 2^32, seed >> 32) and counter
    (j // 4, i, b*H + h, offset) for query i and key j of the sequence; word
    j % 4 of that call is element (i, j)'s draw.
    """
    from .philox import philox4x32_10
    i = np.arange(nq, dtype=np.uint64)[:, None]
    j = np.arange(nk, dtype=np.uint64)[None, :]
    words = philox4x32_10(j >> np.uint64(2), i, np.uint64(b * H + h), np.uint64(offset),
                          np.uint64(seed & 0xFFFFFFFF), np.uint64((seed >> 32) & 0xFFFFFFFF))
    w = np.choose((j & np.uint64(3)).astype(np.int64) + np.zeros((nq, 1), dtype=np.int64), words)
    return w >= np.uint32(dropout_threshold(p))


def attention_forward_dropout(q, k, v, scale: float, causal: bool, p: float, seed: int, offset: int = 0):
    """O = (P o Z) V with Z = keep / (1 - p) elementwise (inverted dropout on
    the attention probabilities), and the LSE of the undropped softmax, fp64.
    The keep mask is dropout_keep()'s."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    B, N, H, d = q.shape
    o = np.empty((B, N, H, d))
    lse = np.empty((B, H, N))
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            pr, lse_rows = _softmax_rows(_scores(q[b, :, h], k[b, :, h], scale, rows, causal))
            z = dropout_keep(b, h, H, N, N, p, seed, offset) / (1.0 - p)
            o[b, :, h] = (pr * z) @ v[b, :, h]
            lse[b, h] = lse_rows
    return o, lse


def attention_backward_dropout(q, k, v, do, scale: float, causal: bool, p: float, seed: int, offset: int = 0):
    """Gradients of attention_forward_dropout (the mask does not depend on the
    inputs): dV = (P o Z)^T dO, dP = (dO V^T) o Z, D_i = sum_j P_ij dP_ij
    (= rowsum(dO o O)), dS = P o (dP - D), dQ = scale dS K, dK = scale dS^T Q.
    Returns dQ, dK, dV [B, N, H, d] and D [B, H, N]."""
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    B, N, H, d = q.shape
    dq, dk, dv = (np.empty((B, N, H, d)) for _ in range(3))
    dd = np.empty((B, H, N))
    rows = np.arange(N)
    for b in range(B):
        for h in range(H):
            qh, kh, vh, doh = q[b, :, h], k[b, :, h], v[b, :, h], do[b, :, h]
            pr, _ = _softmax_rows(_scores(qh, kh, scale, rows, causal))
            z = dropout_keep(b, h, H, N, N, p, seed, offset) / (1.0 - p)
            dv[b, :, h] = (pr * z).T @ doh
            dp = (doh @ vh.T) * z
            drow = (pr * dp).sum(axis=1)
            ds = pr * (dp - drow[:, None])
            dq[b, :, h] = scale * (ds @ kh)
            dk[b, :, h] = scale * (ds.T @ qh)
            dd[b, h] = drow
    return dq, dk, dv, dd

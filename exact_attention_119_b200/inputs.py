"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

This module holds no attention arithmetic. It only draws numbers:

* ``splitmix64`` (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; the 64-bit finaliser as published by Vigna) is used
  as a counter-based generator: element pair ``p`` of stream ``s`` under seed
  ``seed`` hashes the counter ``base(seed, s) + 2p`` and ``+ 2p + 1``.
* The two 53-bit uniforms ``u1 in (0, 1]`` and ``u2 in [0, 1)`` become two
  standard normals by the Box-Muller transform (Box and Muller, 1958):
  ``r = sqrt(-2 ln u1)``, ``z0 = r cos(2 pi u2)``, ``z1 = r sin(2 pi u2)``.
* The fp64 normal is multiplied by ``sigma``, rounded to fp32 (RNE) and then to
  the storage dtype (fp16 or bf16, RNE).

Stream ids: Q = 0, K = 1, V = 2, dO = 3. Seed 0 unless a test says otherwise.
Layout is always the attention layout ``[batch, seqlen, heads, head_dim]``.

The same bits are handed to the GPU (as a torch tensor) and, upcast exactly to
fp64, to the oracle.
"""

from __future__ import annotations

import numpy as np

STREAM_Q = 0
STREAM_K = 1
STREAM_V = 2
STREAM_DO = 3

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def splitmix64(x: np.ndarray) -> np.ndarray:
    """The splitmix64 output function applied to counters ``x`` (uint64)."""
    with np.errstate(over="ignore"):
        z = x + _GOLDEN
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def _stream_base(seed: int, stream: int) -> np.uint64:
    # Disjoint counter ranges per (seed, stream): the stream id sits in the top
    # byte, the seed is mixed below it. Tensors here hold < 2^40 elements.
    mixed = int(splitmix64(np.array([seed & 0xFFFFFFFFFFFFFFFF], dtype=np.uint64))[0])
    return np.uint64(((stream & 0xFF) << 56) ^ (mixed & 0x00FFFF0000000000))


def normal_f64(n: int, seed: int, stream: int, sigma: float = 1.0) -> np.ndarray:
    """``n`` i.i.d. N(0, sigma^2) values in fp64 from counters of one stream."""
    pairs = (n + 1) // 2
    base = _stream_base(seed, stream)
    out = np.empty(2 * pairs, dtype=np.float64)
    chunk = 1 << 22
    for p0 in range(0, pairs, chunk):
        p1 = min(pairs, p0 + chunk)
        idx = np.arange(p0, p1, dtype=np.uint64)
        with np.errstate(over="ignore"):
            c = base + (idx << np.uint64(1))
        a = splitmix64(c)
        b = splitmix64(c + np.uint64(1))
        u1 = ((a >> np.uint64(11)).astype(np.float64) + 1.0) * (2.0 ** -53)
        u2 = (b >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)
        r = np.sqrt(-2.0 * np.log(u1))
        t = 2.0 * np.pi * u2
        out[2 * p0:2 * p1:2] = r * np.cos(t)
        out[2 * p0 + 1:2 * p1:2] = r * np.sin(t)
    return out[:n] * sigma


def f32_to_bf16_bits(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 with round-to-nearest-even; returns uint16 bit patterns."""
    bits = x32.astype(np.float32).view(np.uint32)
    lsb = (bits >> np.uint32(16)) & np.uint32(1)
    with np.errstate(over="ignore"):
        rounded = bits + np.uint32(0x7FFF) + lsb
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    return (u16.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def f16_bits_to_f64(u16: np.ndarray) -> np.ndarray:
    return u16.view(np.float16).astype(np.float64)


def make_tensor_bits(shape, dtype: str, seed: int, stream: int, sigma: float = 1.0) -> np.ndarray:
    """Storage bits (uint16) of one synthetic tensor of ``shape`` in ``dtype``."""
    if dtype not in ("fp16", "bf16"):
        raise ValueError(f"dtype must be 'fp16' or 'bf16', got {dtype!r}")
    n = int(np.prod(shape))
    x32 = normal_f64(n, seed, stream, sigma).astype(np.float32)
    if dtype == "fp16":
        bits = x32.astype(np.float16).view(np.uint16)
    else:
        bits = f32_to_bf16_bits(x32)
    return bits.reshape(shape)


def bits_to_f64(bits: np.ndarray, dtype: str) -> np.ndarray:
    """Exact fp64 values of stored fp16/bf16 bits (what the oracle consumes)."""
    return f16_bits_to_f64(bits) if dtype == "fp16" else bf16_bits_to_f64(bits)


def bits_to_torch(bits: np.ndarray, dtype: str):
    """A CPU torch tensor holding the same bits in torch.float16 / torch.bfloat16."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.float16 if dtype == "fp16" else torch.bfloat16)


def attention_inputs(B: int, N: int, H: int, d: int, dtype: str, seed: int = 0,
                     sigma_qk: float = 1.0, sigma_vdo: float = 1.0, with_do: bool = True):
    """Bits of Q, K, V (and dO) for one workload, each ``[B, N, H, d]``."""
    shape = (B, N, H, d)
    out = {
        "q": make_tensor_bits(shape, dtype, seed, STREAM_Q, sigma_qk),
        "k": make_tensor_bits(shape, dtype, seed, STREAM_K, sigma_qk),
        "v": make_tensor_bits(shape, dtype, seed, STREAM_V, sigma_vdo),
    }
    if with_do:
        out["do"] = make_tensor_bits(shape, dtype, seed, STREAM_DO, sigma_vdo)
    return out

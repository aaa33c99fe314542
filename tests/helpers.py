"""Shared test plumbing: seeded inputs for both sides and error metrics."""

import math

import numpy as np

from exact_attention_119_b200 import inputs

# Tolerances stated for this path: O max-abs, LSE max-abs, gradient relative
# Frobenius error.
O_TOL = {"fp16": 4e-3, "bf16": 1.6e-2}
LSE_TOL = 1e-4
GRAD_REL_TOL = 1e-2


class Case:
    """One seeded workload: storage bits, fp64 copies, and torch tensors."""

    def __init__(self, B, N, H, d, dtype, causal, seed=0, sigma_qk=1.0, with_do=True):
        self.B, self.N, self.H, self.d = B, N, H, d
        self.dtype, self.causal = dtype, causal
        self.scale = 1.0 / math.sqrt(d)
        self.bits = inputs.attention_inputs(B, N, H, d, dtype, seed, sigma_qk=sigma_qk, with_do=with_do)
        self.f64 = {k: inputs.bits_to_f64(v, dtype) for k, v in self.bits.items()}

    def torch(self, name, device="cuda"):
        return inputs.bits_to_torch(self.bits[name], self.dtype).to(device)

    def __repr__(self):
        return f"Case(B={self.B}, N={self.N}, H={self.H}, d={self.d}, {self.dtype}, causal={self.causal})"


def max_abs(a, b):
    return float(np.max(np.abs(np.asarray(a, dtype=np.float64) - np.asarray(b, dtype=np.float64))))


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def sample_rows(N, count=64, seed=0):
    """Rows 0, 1, N-1, every 128-row tile boundary, plus seeded random rows."""
    rows = {0, 1, N - 1}
    for t in range(128, N, 128):
        rows.update({t - 1, t})
    rng = np.random.default_rng(seed)
    rows.update(rng.integers(0, N, size=count).tolist())
    return np.array(sorted(r for r in rows if 0 <= r < N), dtype=np.int64)

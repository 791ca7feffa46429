"""Shared helpers of the GPU parity tests: seeded inputs on the device, the
oracle on matching fp64 slices, and the error metrics with their tolerances.

Tolerances (fixed by the accuracy target of the work): max |O - O_ref| <= 1e-2,
max |LSE - LSE_ref| <= 1e-3, relative L2 error of dQ, dK, dV <= 2e-2.
"""
from __future__ import annotations

import math

import numpy as np

from exact_attention_159_b200 import inputs as I
from oracle import oracle as OR

TOL_O = 1e-2
TOL_LSE = 1e-3
TOL_GRAD = 2e-2


def to_dev(bits: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def bf16_to_f64(t) -> np.ndarray:
    import torch
    return I.bf16_bits_to_f64(t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16))


def sample_rows(N: int, count: int, seed: int) -> np.ndarray:
    """Rows to compare: both ends, the rows on either side of tile boundaries spread evenly over the
    whole length, then seeded random rows up to `count` in all (the fixed rows are always kept)."""
    fixed = {0, 1, 2, N - 1, N - 2}
    bounds = list(range(128, N, 128))
    pairs = max(count // 2 - len(fixed), 0) // 2
    if bounds and pairs:
        step = -(-len(bounds) // pairs)
        for t in bounds[::step]:
            fixed.update((t - 1, t))
    fixed = np.array(sorted(x for x in fixed if 0 <= x < N), dtype=np.int64)
    rest = np.setdiff1d(np.arange(N, dtype=np.int64), fixed)
    n_rnd = max(0, min(count - len(fixed), len(rest)))
    rnd = np.random.default_rng(seed).choice(rest, size=n_rnd, replace=False) if n_rnd else rest[:0]
    return np.unique(np.concatenate([fixed, rnd.astype(np.int64)]))


def rel_l2(a, b) -> float:
    den = float(np.linalg.norm(b))
    return float(np.linalg.norm(a - b)) / (den if den > 0 else 1.0)


class Case:
    """One workload: bf16 bits on the host, device tensors, fp64 views for the oracle."""

    def __init__(self, B, H, N, d, causal, *, seed_workload=9, stress=False, bwd=False):
        import torch
        self.B, self.H, self.N, self.d, self.causal = B, H, N, d, causal
        self.scale = 1.0 / math.sqrt(d)
        self.bits = I.attention_inputs(seed_workload, B, H, N, d, stress=stress, with_do=bwd)
        self.dev = {k: to_dev(v) for k, v in self.bits.items()}
        self.torch = torch

    def head(self, name, b, h):
        return I.bf16_bits_to_f64(self.bits[name][b, h])

    def fwd_gpu(self):
        from exact_attention_159_b200 import api
        o, lse = api.fa_fwd(self.dev["q"], self.dev["k"], self.dev["v"], self.scale, self.causal)
        return o, lse

    def bwd_gpu(self, o, lse):
        from exact_attention_159_b200 import api
        return api.fa_bwd(self.dev["q"], self.dev["k"], self.dev["v"], o, self.dev["do"], lse, self.scale,
                          self.causal)

    def oracle_fwd(self, b, h, rows=None):
        return OR.fwd(self.head("q", b, h), self.head("k", b, h), self.head("v", b, h), self.scale, self.causal,
                      rows=rows)

    def oracle_bwd(self, b, h, qrows=None, krows=None):
        return OR.bwd(self.head("q", b, h), self.head("k", b, h), self.head("v", b, h), self.head("do", b, h),
                      self.scale, self.causal, qrows=qrows, krows=krows)

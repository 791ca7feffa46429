"""Seeded synthetic inputs for exact attention (shared by the CUDA path, the
oracle-based tests and the benchmark).

This module holds none of the attention arithmetic: it only draws numbers.

Recipe (one stream per tensor):
  * counter-based splitmix64: the k-th 64-bit draw of stream ``seed`` is
    ``mix64(seed * 2**32 + k + 1)`` with the standard splitmix64 finaliser
    (Steele, Lea, Flood, "Fast splittable pseudorandom number generators",
    OOPSLA 2014), so any slice of a tensor can be regenerated on its own;
  * uniform doubles ``u = (z >> 11) * 2**-53`` in [0, 1);
  * standard normals by Box-Muller on consecutive pairs (2k, 2k+1), in fp64;
  * fp64 -> fp32 (round to nearest) -> bf16 (round to nearest even).

Seeds: workload ``c`` uses ``seed = 1000 * c + tensor_id`` with tensor ids
Q=0, K=1, V=2, dO=3, direction u=4, offsets=5.

The rescale-stress workload adds, along one random unit direction ``u``, an
offset ``a_i ~ U(0, 8)`` to every query row and ``b_j ~ U(0, 8)`` to every key
row, so that the logits gain ``a_i * b_j * scale`` and row maxima jump from one
key tile to the next (FlashAttention-4 pages, "adaptive online softmax
rescaling" in "The Technical Edge").
"""
from __future__ import annotations

import numpy as np

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "do": 3, "u": 4, "offsets": 5}

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix64(z: np.ndarray) -> np.ndarray:
    z = z * _GOLDEN
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def uniform(seed: int, start: int, count: int) -> np.ndarray:
    """``count`` fp64 uniforms in [0, 1) from draws ``start .. start+count-1`` of stream ``seed``."""
    base = np.uint64((seed & 0xFFFFFFFF) << 32)
    ctr = np.arange(start + 1, start + count + 1, dtype=np.uint64) + base
    with np.errstate(over="ignore"):
        z = _mix64(ctr)
    return (z >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def normal(seed: int, count: int, start: int = 0) -> np.ndarray:
    """``count`` fp64 standard normals of stream ``seed`` (Box-Muller, fp64), starting at normal
    number ``start`` of the stream (even, so that Box-Muller pairs stay aligned)."""
    if start % 2:
        raise ValueError("start must be even")
    out = np.empty(count, dtype=np.float64)
    pairs = (count + 1) // 2
    for p0 in range(0, pairs, _CHUNK):
        p1 = min(pairs, p0 + _CHUNK)
        u = uniform(seed, start + 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
        r = np.sqrt(-2.0 * np.log1p(-u[:, 0]))  # 1 - u in (0, 1]
        t = 2.0 * np.pi * u[:, 1]
        z = np.stack([r * np.cos(t), r * np.sin(t)], axis=1).reshape(-1)
        n = min(count, 2 * p1) - 2 * p0
        out[2 * p0: 2 * p0 + n] = z[:n]
    return out


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp64 -> fp32 (nearest) -> bf16 bit patterns (nearest even), as uint16."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    b = b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
    return (b >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp64."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def seed_for(workload: int, tensor: str) -> int:
    return 1000 * workload + TENSOR_IDS[tensor]


def normal_bf16(seed: int, shape) -> np.ndarray:
    """bf16 bit patterns (uint16) of i.i.d. N(0, 1) draws with the given shape."""
    n = int(np.prod(shape))
    return f64_to_bf16_bits(normal(seed, n)).reshape(shape)


def attention_inputs(workload: int, B: int, H: int, N: int, d: int, *,
                     stress: bool = False, with_do: bool = False) -> dict:
    """bf16 bit arrays (uint16, shape B x H x N x d) for one workload.

    ``stress`` selects the rescale-stress construction described in the module
    docstring; otherwise every tensor is i.i.d. N(0, 1).
    """
    shape = (B, H, N, d)
    out = {}
    if stress:
        u = normal(seed_for(workload, "u"), d)
        u /= np.sqrt(np.sum(u * u))
        rows = B * H * N
        off = uniform(seed_for(workload, "offsets"), 0, 2 * rows) * 8.0
        for name, a in (("q", off[:rows]), ("k", off[rows:])):
            x = normal(seed_for(workload, name), rows * d).reshape(rows, d)
            x += a[:, None] * u[None, :]
            out[name] = f64_to_bf16_bits(x).reshape(shape)
    else:
        out["q"] = normal_bf16(seed_for(workload, "q"), shape)
        out["k"] = normal_bf16(seed_for(workload, "k"), shape)
    out["v"] = normal_bf16(seed_for(workload, "v"), shape)
    if with_do:
        out["do"] = normal_bf16(seed_for(workload, "do"), shape)
    return out


def head_inputs(workload: int, B: int, H: int, N: int, d: int, b: int, h: int, *,
                stress: bool = False, with_do: bool = False) -> dict:
    """The (b, h) slice (N x d bf16 bit arrays) of ``attention_inputs(workload, B, H, N, d, ...)``,
    drawn on its own from the counter-based streams (equal to slicing the full tensors)."""
    row0 = (b * H + h) * N  # first row of this head in the B*H*N rows of each tensor
    out = {}
    if stress:
        u = normal(seed_for(workload, "u"), d)
        u /= np.sqrt(np.sum(u * u))
        rows = B * H * N
        for name, first in (("q", row0), ("k", rows + row0)):
            a = uniform(seed_for(workload, "offsets"), first, N) * 8.0
            x = normal(seed_for(workload, name), N * d, start=row0 * d).reshape(N, d)
            x += a[:, None] * u[None, :]
            out[name] = f64_to_bf16_bits(x)
    else:
        for name in ("q", "k"):
            out[name] = f64_to_bf16_bits(normal(seed_for(workload, name), N * d, start=row0 * d)).reshape(N, d)
    names = ("v", "do") if with_do else ("v",)
    for name in names:
        out[name] = f64_to_bf16_bits(normal(seed_for(workload, name), N * d, start=row0 * d)).reshape(N, d)
    return out


def attention_inputs_qk(workload: int, B: int, Hq: int, Hkv: int, Nq: int, Nk: int, d: int, *,
                        with_do: bool = False) -> dict:
    """bf16 bit arrays (uint16) for grouped-query attention with unequal lengths: q (and do)
    B x Hq x Nq x d, k and v B x Hkv x Nk x d, each i.i.d. N(0, 1) from its own stream."""
    out = {"q": normal_bf16(seed_for(workload, "q"), (B, Hq, Nq, d)),
           "k": normal_bf16(seed_for(workload, "k"), (B, Hkv, Nk, d)),
           "v": normal_bf16(seed_for(workload, "v"), (B, Hkv, Nk, d))}
    if with_do:
        out["do"] = normal_bf16(seed_for(workload, "do"), (B, Hq, Nq, d))
    return out


# The five workloads of the FlashAttention-4 evaluation this library is
# measured on (shapes, causal flag, structure).  Workload 5 is a sweep.
WORKLOADS = {
    1: dict(name="tiny-fwd", B=1, H=1, N=128, d=64, causal=False, stress=False, bwd=False),
    2: dict(name="fwd-causal", B=4, H=16, N=2048, d=128, causal=True, stress=False, bwd=False),
    3: dict(name="fwd-rescale-stress", B=2, H=16, N=8192, d=128, causal=False, stress=True, bwd=False),
    4: dict(name="long-fwd-bwd-causal", B=1, H=16, N=32768, d=128, causal=True, stress=False, bwd=True),
}

# Workload 5: 16384 tokens, H=16, d in {64,128}, both causal modes.
SWEEP = [dict(name=f"bwd-sweep-B{B}-N{N}-d{d}-{'causal' if c else 'full'}",
              B=B, H=16, N=N, d=d, causal=c, stress=False, bwd=True)
         for (B, N) in ((8, 2048), (2, 8192), (1, 16384)) for d in (64, 128) for c in (False, True)]

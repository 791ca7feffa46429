"""Host fp32 emulation of the kernels' software exp2 (same constants, same operation order)."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "exact_attention_159_b200", "csrc", "exp2_poly.cuh")


def coefficients():
    text = open(HDR).read()
    return [np.float32(float(re.search(rf"#define FA_EXP2_C{i} ([-0-9.e+]+)f", text).group(1))) for i in range(4)]


def _fma32(a, b, c):
    # a*b is exact in fp64 for fp32 operands; one rounding of the sum to fp32 models the fused op
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def exp2_poly_f32(x):
    c0, c1, c2, c3 = coefficients()
    x = np.maximum(np.asarray(x, dtype=np.float32), np.float32(-126.0))
    k = np.float32(12582912.0)
    # x + k rounded toward -inf: the exact sum is representable in fp64, so
    # floor(x) + k is what a round-down fp32 add produces here
    t = (np.floor(x.astype(np.float64)) + np.float64(k)).astype(np.float32)
    j = (t - k).astype(np.float32)
    f = (x - j).astype(np.float32)
    p = _fma32(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.full_like(f, c0))
    ji = t.view(np.int32) - np.int32(0x4B400000)
    return (p.view(np.int32) + (ji << 23)).view(np.float32)


def sweep_points(n=1 << 24, lo=-126.0, hi=0.0):
    x = np.linspace(lo, hi, n, dtype=np.float64).astype(np.float32)
    ints = np.arange(int(lo), int(hi) + 1, dtype=np.float32)
    nb = np.concatenate([np.nextafter(ints, np.float32(-np.inf)), np.nextafter(ints, np.float32(np.inf)),
                         ints + np.float32(0.5), np.nextafter(ints + np.float32(0.5), np.float32(np.inf)),
                         np.nextafter(ints + np.float32(0.5), np.float32(-np.inf))]).astype(np.float32)
    x = np.concatenate([x, ints, nb])
    return x[(x >= lo) & (x <= hi)]

"""The cubic software exp2, emulated in fp32 on the host, against fp64 exp2 (a closed form)."""
import numpy as np

from tests.exp2_host import exp2_poly_f32, sweep_points


def test_sweep_relative_error():
    x = sweep_points()
    y = exp2_poly_f32(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(y / ref - 1.0)
    assert rel.max() <= 2e-4, rel.max()
    assert rel.max() <= 9e-5       # the minimax bound (8.6e-5) plus fp32 rounding


def test_exact_at_integers():
    # p(0) = 1 is pinned, so integer x give exact powers of two, down to 2^-126
    n = np.arange(-126, 9, dtype=np.float32)
    assert np.array_equal(exp2_poly_f32(n).astype(np.float64), np.exp2(n.astype(np.float64)))


def test_positive_range_and_clamp():
    x = np.linspace(0.0, 8.0, 100001, dtype=np.float32)     # P <= 2^tau with tau = 8
    rel = np.abs(exp2_poly_f32(x).astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 9e-5
    low = exp2_poly_f32(np.array([-127.0, -200.0, -np.inf], dtype=np.float32)).astype(np.float64)
    assert np.all(low >= 0.0) and np.all(low == 2.0 ** -126)

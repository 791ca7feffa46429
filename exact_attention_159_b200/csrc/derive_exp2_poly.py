"""Derive the cubic used by the kernels' software exp2 (prints C constants).

The FlashAttention-4 pages ("The Technical Edge"; "B. Remplacer le Couteau
Lourd") say the exponential is emulated on the FMA units with a cubic
polynomial but give no coefficients or range reduction.  Ours:

    x = j + f,  j = floor(x),  f in [0, 1)
    2^x ~= p(f) * 2^j,  p(f) = 1 + c1 f + c2 f^2 + c3 f^3

p(0) = 1 is pinned so that p(f) >= 1 on [0, 1): the result then stays a
normal fp32 number down to x = -126, and integer x give exact powers of two.
c1..c3 minimise the maximum RELATIVE error |p(f)/2^f - 1| on [0, 1] (Remez
exchange, 4 alternation points, fp64).  The scaling by 2^j is an integer add
into the fp32 exponent field.

Run:  python derive_exp2_poly.py
"""
import numpy as np


def remez_relative_pinned(lo=0.0, hi=1.0, iters=40):
    f = np.exp2
    n_free = 3                      # c1, c2, c3
    n = n_free + 1                  # alternation points
    x = lo + (hi - lo) * 0.5 * (1 - np.cos(np.pi * (np.arange(n) + 0.5) / n))
    grid = np.linspace(lo, hi, 400001)
    c = None
    for _ in range(iters):
        # 1 + sum_k c_k x^k - f(x) = (-1)^i E f(x)   for the n reference points
        A = np.zeros((n, n))
        for i in range(n):
            A[i, :n_free] = x[i] ** np.arange(1, n_free + 1)
            A[i, n_free] = -((-1) ** i) * f(x[i])
        sol = np.linalg.solve(A, f(x) - 1.0)
        c = np.concatenate([[1.0], sol[:n_free]])
        err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
        sgn = np.sign(err)
        idx = np.where(np.diff(sgn) != 0)[0]
        bounds = np.concatenate([[0], idx + 1, [len(grid)]])
        ext = [b0 + np.argmax(np.abs(err[b0:b1])) for b0, b1 in zip(bounds[:-1], bounds[1:]) if b1 > b0]
        # keep the n largest alternating extrema (the pinned end at 0 has zero error)
        ext = [e for e in ext if grid[e] > lo] if len(ext) > n else ext
        if len(ext) != n:
            break
        x = grid[ext]
    err = (np.polyval(c[::-1], grid) - f(grid)) / f(grid)
    return c, float(np.max(np.abs(err)))


if __name__ == "__main__":
    c, e = remez_relative_pinned()
    print("// minimax cubic for 2^f on [0, 1), p(0) = 1; max relative error %.3e" % e)
    for i, v in enumerate(np.float32(c)):
        print(f"#define FA_EXP2_C{i} {float(v):.9e}f")

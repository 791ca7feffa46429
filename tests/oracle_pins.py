"""Pins for the fp64 attention oracle: checks against things other than the
oracle itself (a hand-worked example, closed forms, invariants, finite
differences, and torch's own fp64 attention + autograd on tiny inputs).

Each pin takes the ctypes oracle library so the mutation test can run the same
pins against copies of the oracle with a mistake planted in them.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64); b = np.asarray(b, dtype=np.float64)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert np.all(np.isfinite(a)), f"{what}: non-finite values"
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


def _val(x):
    if isinstance(x, (int, float)):
        return float(x)
    table = {"ln3": math.log(3.0), "ln4": math.log(4.0), "ln10": math.log(10.0),
             "0.75*ln3": 0.75 * math.log(3.0), "0.36*ln3": 0.36 * math.log(3.0)}
    return table[x]


def _arr(x):
    return np.array([[_val(e) for e in row] if isinstance(row, list) else _val(row) for row in x],
                    dtype=np.float64)


# --------------------------------------------------------------------- pins
def pin_golden_worked_example(lib):
    """Hand-derived two-key example (tests/golden/worked_example_two_keys.json)."""
    g = json.load(open(os.path.join(GOLDEN, "worked_example_two_keys.json")))
    q, k, v, do = (_arr(g["inputs"][n]) for n in ("q", "k", "v", "dO"))
    sc = g["inputs"]["scale"]
    for mode, causal in (("full", False), ("causal", True)):
        exp = g[mode]
        o, lse = O.fwd(q, k, v, sc, causal, nthreads=2, lib=lib)
        _close(o, _arr(exp["O"]), 1e-13, f"golden {mode} O")
        _close(lse, _arr(exp["LSE"]), 1e-13, f"golden {mode} LSE")
        dq, dk, dv, _, _ = O.bwd(q, k, v, do, sc, causal, nthreads=2, lib=lib)
        _close(dq, _arr(exp["dQ"]), 1e-13, f"golden {mode} dQ")
        _close(dk, _arr(exp["dK"]), 1e-13, f"golden {mode} dK")
        _close(dv, _arr(exp["dV"]), 1e-13, f"golden {mode} dV")


def pin_torch_library(lib):
    """torch fp64 scaled_dot_product_attention + autograd (independent library)."""
    import torch
    for (n, d, causal, seed) in ((1, 4, False, 1), (5, 3, True, 2), (17, 8, False, 3),
                                 (33, 16, True, 4), (64, 32, True, 5), (40, 24, False, 6)):
        r = _rng(seed)
        q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
        scale = 1.0 / math.sqrt(d) * (1.0 + 0.5 * seed)
        t = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q, k, v)]
        ref = torch.nn.functional.scaled_dot_product_attention(t[0][None], t[1][None], t[2][None],
                                                               is_causal=causal, scale=scale)[0]
        ref.backward(torch.tensor(do))
        o, lse = O.fwd(q, k, v, scale, causal, nthreads=3, lib=lib)
        _close(o, ref.detach().numpy(), 1e-12, f"torch O n={n}")
        s = scale * (q @ k.T)
        if causal:
            s = np.where(np.tril(np.ones((n, n), bool)), s, -np.inf)
        lse_t = torch.logsumexp(torch.tensor(s), dim=1).numpy()
        _close(lse, lse_t, 1e-12, f"torch logsumexp n={n}")
        dq, dk, dv, lse2, _ = O.bwd(q, k, v, do, scale, causal, nthreads=3, lib=lib)
        _close(lse2, lse_t, 1e-12, f"bwd LSE n={n}")
        for a, b, nm in ((dq, t[0].grad, "dQ"), (dk, t[1].grad, "dK"), (dv, t[2].grad, "dV")):
            _close(a, b.numpy(), 1e-11, f"torch {nm} n={n}")


def pin_zero_query(lib):
    """Q = 0: every visible key weighs the same -> O_i = mean of visible V, LSE_i = ln(#visible)."""
    n, d = 37, 12
    r = _rng(11)
    k, v = r.standard_normal((n, d)), r.standard_normal((n, d))
    q = np.zeros((n, d))
    for causal in (False, True):
        o, lse = O.fwd(q, k, v, 0.3, causal, nthreads=2, lib=lib)
        cnt = np.arange(1, n + 1) if causal else np.full(n, n)
        mean = np.cumsum(v, axis=0) / cnt[:, None] if causal else np.broadcast_to(v.mean(0), (n, d))
        _close(o, mean, 1e-13, f"Q=0 O causal={causal}")
        _close(lse, np.log(cnt), 1e-13, f"Q=0 LSE causal={causal}")


def pin_single_key(lib):
    """N = 1: O = V, LSE = scale q.k, dQ = dK = 0, dV = dO."""
    r = _rng(12)
    for d in (1, 7, 64):
        q, k, v, do = (r.standard_normal((1, d)) for _ in range(4))
        for causal in (False, True):
            o, lse = O.fwd(q, k, v, 0.7, causal, nthreads=1, lib=lib)
            _close(o, v, 1e-14, "N=1 O")
            _close(lse, [0.7 * float(q[0] @ k[0])], 1e-13, "N=1 LSE")
            dq, dk, dv, _, _ = O.bwd(q, k, v, do, 0.7, causal, nthreads=1, lib=lib)
            _close(dq, 0 * dq, 1e-14, "N=1 dQ")
            _close(dk, 0 * dk, 1e-14, "N=1 dK")
            _close(dv, do, 1e-14, "N=1 dV")


def pin_constant_values(lib):
    """All V rows equal to one vector c: O_i = c; the softmax gradient vanishes, dQ = dK = 0."""
    n, d = 29, 10
    r = _rng(13)
    q, k, do = (r.standard_normal((n, d)) for _ in range(3))
    c = r.standard_normal(d)
    v = np.tile(c, (n, 1))
    for causal in (False, True):
        o, _ = O.fwd(q, k, v, 0.4, causal, nthreads=2, lib=lib)
        _close(o, np.tile(c, (n, 1)), 1e-13, "constant V -> O")
        dq, dk, dv, _, _ = O.bwd(q, k, v, do, 0.4, causal, nthreads=2, lib=lib)
        _close(dq, 0 * dq, 1e-12, "constant V -> dQ")
        _close(dk, 0 * dk, 1e-12, "constant V -> dK")


def pin_dominant_logit(lib):
    """One key with a logit 40 above the rest: O_i ~= that key's V row, LSE_i ~= its logit."""
    n, d = 24, 8
    r = _rng(14)
    k = 0.01 * r.standard_normal((n, d))
    v = r.standard_normal((n, d))
    jstar = 5
    k[jstar, :] = 0.0
    k[jstar, 0] = 40.0
    q = np.zeros((n, d)); q[:, 0] = 1.0
    o, lse = O.fwd(q, k, v, 1.0, False, nthreads=2, lib=lib)
    _close(o, np.tile(v[jstar], (n, 1)), 1e-14, "dominant logit O")
    _close(lse, np.full(n, 40.0), 1e-14, "dominant logit LSE")


def pin_rows_sum_to_one(lib):
    """V = all ones: O_i = sum_j P_ij = 1 for every row."""
    n, d = 45, 9
    r = _rng(15)
    q, k = 3 * r.standard_normal((n, d)), 3 * r.standard_normal((n, d))
    for causal in (False, True):
        o, _ = O.fwd(q, k, np.ones((n, d)), 0.5, causal, nthreads=4, lib=lib)
        _close(o, np.ones((n, d)), 1e-13, "rows sum to 1")


def pin_key_shift(lib):
    """Adding w to every key: O unchanged, LSE_i shifted by scale q_i . w (softmax shift invariance)."""
    n, d, sc = 31, 6, 0.45
    r = _rng(16)
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    w = r.standard_normal(d)
    for causal in (False, True):
        o1, l1 = O.fwd(q, k, v, sc, causal, nthreads=2, lib=lib)
        o2, l2 = O.fwd(q, k + w, v, sc, causal, nthreads=2, lib=lib)
        _close(o2, o1, 1e-12, "key shift O")
        _close(l2 - l1, sc * (q @ w), 1e-12, "key shift LSE")


def pin_permutation(lib):
    """Non-causal: permuting keys and values together leaves O, LSE unchanged; permuting queries permutes rows."""
    n, d = 26, 5
    r = _rng(17)
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    p = r.permutation(n)
    o1, l1 = O.fwd(q, k, v, 0.6, False, nthreads=2, lib=lib)
    o2, l2 = O.fwd(q, k[p], v[p], 0.6, False, nthreads=2, lib=lib)
    _close(o2, o1, 1e-13, "key permutation O")
    _close(l2, l1, 1e-13, "key permutation LSE")
    o3, l3 = O.fwd(q[p], k, v, 0.6, False, nthreads=2, lib=lib)
    _close(o3, o1[p], 1e-13, "query permutation O")


def pin_causal_prefix(lib):
    """Causal row i equals the non-causal result on the first i+1 keys and values."""
    n, d = 20, 4
    r = _rng(18)
    q, k, v = (r.standard_normal((n, d)) for _ in range(3))
    o, lse = O.fwd(q, k, v, 0.8, True, nthreads=2, lib=lib)
    for i in (0, 1, 7, 19):
        qq = np.zeros((i + 1, d))
        qq[0] = q[i]
        oi, li = O.fwd(qq, k[:i + 1], v[:i + 1], 0.8, False, rows=[0], nthreads=1, lib=lib)
        _close(oi[0], o[i], 1e-13, f"causal prefix O row {i}")
        _close(li, [lse[i]], 1e-13, f"causal prefix LSE row {i}")


def pin_gradient_sums(lib):
    """sum_j dK_j = 0 (softmax shift invariance) and sum_j dV_j = sum_i dO_i (rows sum to 1)."""
    n, d = 33, 7
    r = _rng(19)
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    for causal in (False, True):
        dq, dk, dv, _, _ = O.bwd(q, k, v, do, 0.5, causal, nthreads=3, lib=lib)
        _close(dk.sum(0), np.zeros(d), 1e-12, "sum dK = 0")
        _close(dv.sum(0), do.sum(0), 1e-12, "sum dV = sum dO")


def pin_finite_differences(lib):
    """Central differences of L = sum(dO * O) w.r.t. Q, K, V (h = 1e-6) match dQ, dK, dV."""
    n, d, sc, h = 9, 5, 0.55, 1e-6
    r = _rng(20)
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    for causal in (False, True):
        dq, dk, dv, _, _ = O.bwd(q, k, v, do, sc, causal, nthreads=2, lib=lib)

        def L(qq, kk, vv):
            o, _ = O.fwd(qq, kk, vv, sc, causal, nthreads=2, lib=lib)
            return float(np.sum(do * o))

        for which, g in ((0, dq), (1, dk), (2, dv)):
            num = np.zeros((n, d))
            for i in range(n):
                for c in range(d):
                    args_p = [q.copy(), k.copy(), v.copy()]
                    args_m = [q.copy(), k.copy(), v.copy()]
                    args_p[which][i, c] += h
                    args_m[which][i, c] -= h
                    num[i, c] = (L(*args_p) - L(*args_m)) / (2 * h)
            rel = np.linalg.norm(num - g) / max(np.linalg.norm(g), 1e-30)
            assert rel < 1e-7, f"finite differences operand {which} causal={causal}: rel {rel:.2e}"


def pin_row_subsets(lib):
    """Row-sampled forward / backward equal the corresponding rows of the full computation."""
    n, d = 50, 8
    r = _rng(21)
    q, k, v, do = (r.standard_normal((n, d)) for _ in range(4))
    rows = np.array([0, 3, 17, 49, 25])
    for causal in (False, True):
        o, lse = O.fwd(q, k, v, 0.5, causal, nthreads=3, lib=lib)
        os_, ls_ = O.fwd(q, k, v, 0.5, causal, rows=rows, nthreads=2, lib=lib)
        _close(os_, o[rows], 0.0, "row subset O")
        _close(ls_, lse[rows], 0.0, "row subset LSE")
        dq, dk, dv, _, _ = O.bwd(q, k, v, do, 0.5, causal, nthreads=3, lib=lib)
        dqs, dks, dvs, _, _ = O.bwd(q, k, v, do, 0.5, causal, qrows=rows, krows=rows[::-1],
                                    nthreads=5, lib=lib)
        _close(dqs, dq[rows], 0.0, "row subset dQ")
        _close(dks, dk[rows[::-1]], 0.0, "row subset dK")
        _close(dvs, dv[rows[::-1]], 0.0, "row subset dV")


def _torch_masked(q, k, v, do, scale, causal, rows):
    """torch fp64 attention with an explicit boolean mask (the last query aligned with the last
    key) over the query ``rows`` that see at least one key, with autograd gradients."""
    import torch
    nq, nk = q.shape[0], k.shape[0]
    i = np.asarray(rows)[:, None]
    j = np.arange(nk)[None, :]
    mask = (j <= i + (nk - nq)) if causal else np.ones((len(rows), nk), bool)
    t = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (q[rows], k, v)]
    ref = torch.nn.functional.scaled_dot_product_attention(t[0][None], t[1][None], t[2][None],
                                                           attn_mask=torch.tensor(mask)[None], scale=scale)[0]
    ref.backward(torch.tensor(do[rows]))
    s = np.where(mask, scale * (q[rows] @ k.T), -np.inf)
    lse = torch.logsumexp(torch.tensor(s), dim=1).numpy()
    return ref.detach().numpy(), lse, t[0].grad.numpy(), t[1].grad.numpy(), t[2].grad.numpy()


def pin_torch_rectangular(lib):
    """nq != nk, causal aligned bottom-right: torch fp64 attention with an explicit mask + autograd
    over the rows that see a key; the rows that see none are O = 0, LSE = -inf, dQ = 0 and add
    nothing to dK, dV (so torch over the visible rows alone gives the same dK, dV)."""
    for (nq, nk, d, causal, seed) in ((5, 11, 4, True, 31), (11, 5, 4, True, 32), (7, 13, 6, False, 33),
                                      (1, 9, 3, True, 34), (16, 40, 8, True, 35), (40, 16, 8, True, 36)):
        r = _rng(seed)
        q, do = r.standard_normal((nq, d)), r.standard_normal((nq, d))
        k, v = r.standard_normal((nk, d)), r.standard_normal((nk, d))
        scale = 0.7 / math.sqrt(d)
        seen = np.arange(nq) + (nk - nq) >= 0 if causal else np.ones(nq, bool)
        rows = np.nonzero(seen)[0]
        o_t, lse_t, dq_t, dk_t, dv_t = _torch_masked(q, k, v, do, scale, causal, rows)
        o, lse = O.fwd(q, k, v, scale, causal, nthreads=3, lib=lib)
        _close(o[rows], o_t, 1e-12, f"rect O {nq}x{nk}")
        _close(lse[rows], lse_t, 1e-12, f"rect LSE {nq}x{nk}")
        dq, dk, dv, lse2, _ = O.bwd(q, k, v, do, scale, causal, nthreads=2, lib=lib)
        _close(dq[rows], dq_t, 1e-11, f"rect dQ {nq}x{nk}")
        _close(dk, dk_t, 1e-11, f"rect dK {nq}x{nk}")
        _close(dv, dv_t, 1e-11, f"rect dV {nq}x{nk}")
        blind = np.nonzero(~seen)[0]
        if blind.size:
            _close(o[blind], np.zeros((blind.size, d)), 0.0, "masked rows O = 0")
            _close(dq[blind], np.zeros((blind.size, d)), 0.0, "masked rows dQ = 0")
            assert np.all(np.isneginf(lse[blind])) and np.all(np.isneginf(lse2[blind])), "masked rows LSE = -inf"


def pin_cache_suffix(lib):
    """Causal nq < nk (new queries over a cache of earlier keys) equals the last nq rows of the
    square causal problem whose last nq queries are those; with the earlier rows' dO = 0 the
    square problem's dK, dV equal the rectangular ones."""
    nq, nk, d = 6, 15, 5
    r = _rng(37)
    qfull, dofull = r.standard_normal((nk, d)), r.standard_normal((nk, d))
    dofull[: nk - nq] = 0.0
    k, v = r.standard_normal((nk, d)), r.standard_normal((nk, d))
    q, do = qfull[nk - nq:], dofull[nk - nq:]
    o, lse = O.fwd(q, k, v, 0.6, True, nthreads=2, lib=lib)
    of, lf = O.fwd(qfull, k, v, 0.6, True, nthreads=2, lib=lib)
    _close(o, of[nk - nq:], 1e-13, "cache suffix O")
    _close(lse, lf[nk - nq:], 1e-13, "cache suffix LSE")
    dq, dk, dv, _, _ = O.bwd(q, k, v, do, 0.6, True, nthreads=2, lib=lib)
    dqf, dkf, dvf, _, _ = O.bwd(qfull, k, v, dofull, 0.6, True, nthreads=3, lib=lib)
    _close(dq, dqf[nk - nq:], 1e-13, "cache suffix dQ")
    _close(dk, dkf, 1e-13, "cache suffix dK")
    _close(dv, dvf, 1e-13, "cache suffix dV")


def pin_gqa_torch(lib):
    """Grouped-query attention (Hq query heads over Hkv key/value heads) against torch fp64 with the
    key/value heads repeated per group: autograd sums the gradients of a repeated head."""
    import torch
    for (Hq, Hkv, nq, nk, causal, seed) in ((4, 2, 9, 9, True, 41), (6, 1, 6, 10, True, 42), (4, 4, 7, 7, False, 43),
                                             (8, 2, 12, 5, False, 44)):
        d = 6
        r = _rng(seed)
        Q, dO = r.standard_normal((Hq, nq, d)), r.standard_normal((Hq, nq, d))
        K, V = r.standard_normal((Hkv, nk, d)), r.standard_normal((Hkv, nk, d))
        scale = 1.0 / math.sqrt(d)
        G = Hq // Hkv
        t = [torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V)]
        i = np.arange(nq)[:, None]; j = np.arange(nk)[None, :]
        mask = torch.tensor((j <= i + (nk - nq)) if causal else np.ones((nq, nk), bool))
        ref = torch.nn.functional.scaled_dot_product_attention(
            t[0], t[1].repeat_interleave(G, dim=0), t[2].repeat_interleave(G, dim=0), attn_mask=mask, scale=scale)
        ref.backward(torch.tensor(dO))
        o, _ = O.gqa_fwd(Q, K, V, scale, causal, nthreads=2, lib=lib)
        _close(o, ref.detach().numpy(), 1e-12, f"GQA O {Hq}/{Hkv}")
        dq, dk, dv, _, _ = O.gqa_bwd(Q, K, V, dO, scale, causal, nthreads=2, lib=lib)
        for a, b, nm in ((dq, t[0].grad, "dQ"), (dk, t[1].grad, "dK"), (dv, t[2].grad, "dV")):
            _close(a, b.numpy(), 1e-11, f"GQA {nm} {Hq}/{Hkv}")


PINS = [pin_golden_worked_example, pin_torch_library, pin_zero_query, pin_single_key,
        pin_constant_values, pin_dominant_logit, pin_rows_sum_to_one, pin_key_shift,
        pin_permutation, pin_causal_prefix, pin_gradient_sums, pin_finite_differences,
        pin_row_subsets, pin_torch_rectangular, pin_cache_suffix, pin_gqa_torch]

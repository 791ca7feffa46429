"""Python handle on the fp64 CPU attention oracle (``attn_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  Nothing in the product path imports
this module, and it imports nothing from the product package.

All operands are fp64 numpy arrays of one (batch, head) slice, row-major:
``nq x d`` queries (and dO), ``nk x d`` keys and values (causal masking aligns
the last query with the last key); bf16 inputs are widened exactly to fp64
before they get here.  Grouped-query attention (several query heads sharing
one key/value head) is the plain per-head computation with the shared K and V,
and the gradients of a shared K or V are the sums over its query heads
(``gqa_fwd`` / ``gqa_bwd``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB_DIR = os.path.join(_HERE, "_build")
_LIB = os.path.join(_LIB_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_ip = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle with gcc (portable flags, no -march)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        os.makedirs(os.path.dirname(out), exist_ok=True)
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def load(path: str | None = None):
    """Load (building first if needed) and return the ctypes library."""
    global _lib
    with _lock:
        if path is not None:
            return _bind(ctypes.CDLL(path))
        if _lib is None:
            _lib = _bind(ctypes.CDLL(build()))
        return _lib


def _bind(lib):
    I64, F64 = ctypes.c_int64, ctypes.c_double
    lib.oracle_attn_fwd_qk.restype = ctypes.c_int
    lib.oracle_attn_fwd_qk.argtypes = [_dp, _dp, _dp, I64, I64, I64, F64, ctypes.c_int, _ip, I64, _dp, _dp,
                                       ctypes.c_int]
    lib.oracle_attn_bwd_qk.restype = ctypes.c_int
    lib.oracle_attn_bwd_qk.argtypes = [_dp, _dp, _dp, _dp, I64, I64, I64, F64, ctypes.c_int, _ip, I64, _ip, I64,
                                       _dp, _dp, _dp, _dp, _dp, ctypes.c_int]
    return lib


def default_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:  # pragma: no cover
        return max(1, os.cpu_count() or 1)


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


def _iptr(a):
    return None if a is None else a.ctypes.data_as(_ip)


def fwd(q, k, v, scale: float, causal: bool, rows=None, nthreads: int | None = None, lib=None):
    """Exact forward for one head: returns ``(O, LSE)`` for query ``rows`` (all if None)."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    nq, d = q.shape
    nk = k.shape[0]
    assert k.shape == (nk, d) and v.shape == (nk, d)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    cnt = nq if r is None else r.shape[0]
    o = np.zeros((cnt, d), dtype=np.float64)
    lse = np.zeros(cnt, dtype=np.float64)
    st = lib.oracle_attn_fwd_qk(_ptr(q), _ptr(k), _ptr(v), nq, nk, d, float(scale), int(bool(causal)),
                                _iptr(r), cnt, _ptr(o), _ptr(lse), int(nthreads or default_threads()))
    if st != 0:
        raise RuntimeError(f"oracle_attn_fwd failed ({st})")
    return o, lse


def bwd(q, k, v, do, scale: float, causal: bool, qrows=None, krows=None,
        nthreads: int | None = None, lib=None):
    """Exact backward for one head.

    Returns ``(dQ[qrows], dK[krows], dV[krows], LSE, D)``; ``LSE`` and ``D``
    cover every query row.  ``qrows``/``krows`` None means all rows.
    """
    lib = lib or load()
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    nq, d = q.shape
    nk = k.shape[0]
    assert k.shape == (nk, d) and v.shape == (nk, d) and do.shape == (nq, d)
    qr = None if qrows is None else np.ascontiguousarray(qrows, dtype=np.int64)
    kr = None if krows is None else np.ascontiguousarray(krows, dtype=np.int64)
    cq = nq if qr is None else qr.shape[0]
    ck = nk if kr is None else kr.shape[0]
    dq = np.zeros((cq, d)); dk = np.zeros((ck, d)); dv = np.zeros((ck, d))
    lse = np.zeros(nq); dsum = np.zeros(nq)
    st = lib.oracle_attn_bwd_qk(_ptr(q), _ptr(k), _ptr(v), _ptr(do), nq, nk, d, float(scale), int(bool(causal)),
                                _iptr(qr), cq, _iptr(kr), ck, _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(lse), _ptr(dsum), int(nthreads or default_threads()))
    if st != 0:
        raise RuntimeError(f"oracle_attn_bwd failed ({st})")
    return dq, dk, dv, lse, dsum


def gqa_fwd(Q, K, V, scale: float, causal: bool, rows=None, nthreads: int | None = None, lib=None):
    """Forward of one batch entry with Hq query heads over Hkv = Hq / G key/value heads
    (``Q``: Hq x nq x d, ``K``/``V``: Hkv x nk x d): query head h reads key/value head h // G."""
    Hq, Hkv = Q.shape[0], K.shape[0]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    outs = [fwd(Q[h], K[h // G], V[h // G], scale, causal, rows=rows, nthreads=nthreads, lib=lib) for h in range(Hq)]
    return np.stack([o for o, _ in outs]), np.stack([l for _, l in outs])


def gqa_bwd(Q, K, V, dO, scale: float, causal: bool, qrows=None, krows=None, nthreads: int | None = None,
            lib=None):
    """Backward of one batch entry under grouped-query attention: dQ per query head, and dK, dV of
    each key/value head summed over the G query heads that read it.  Returns dQ, dK, dV, LSE, D."""
    Hq, Hkv = Q.shape[0], K.shape[0]
    assert Hq % Hkv == 0
    G = Hq // Hkv
    dQ, dK, dV, L, Dd = [], [], [], [], []
    for g in range(Hkv):
        acc_k = acc_v = None
        for h in range(g * G, (g + 1) * G):
            dq, dk, dv, lse, dsum = bwd(Q[h], K[g], V[g], dO[h], scale, causal, qrows=qrows, krows=krows,
                                        nthreads=nthreads, lib=lib)
            dQ.append(dq); L.append(lse); Dd.append(dsum)
            acc_k = dk if acc_k is None else acc_k + dk
            acc_v = dv if acc_v is None else acc_v + dv
        dK.append(acc_k); dV.append(acc_v)
    return np.stack(dQ), np.stack(dK), np.stack(dV), np.stack(L), np.stack(Dd)

"""Python handle on the fp64 CPU attention oracle (``attn_oracle.c``).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg are the only callers.  Nothing in the product path imports
this module, and it imports nothing from the product package.

All operands are fp64 numpy arrays of one (batch, head) slice, row-major
``n x d``; bf16 inputs are widened exactly to fp64 before they get here.
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
    lib.oracle_attn_fwd.restype = ctypes.c_int
    lib.oracle_attn_fwd.argtypes = [_dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                    ctypes.c_int, _ip, ctypes.c_int64, _dp, _dp, ctypes.c_int]
    lib.oracle_attn_bwd.restype = ctypes.c_int
    lib.oracle_attn_bwd.argtypes = [_dp, _dp, _dp, _dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_double,
                                    ctypes.c_int, _ip, ctypes.c_int64, _ip, ctypes.c_int64,
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
    """Exact forward for one head: returns ``(O, LSE)`` for ``rows`` (all rows if None)."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    n, d = q.shape
    assert k.shape == (n, d) and v.shape == (n, d)
    r = None if rows is None else np.ascontiguousarray(rows, dtype=np.int64)
    cnt = n if r is None else r.shape[0]
    o = np.zeros((cnt, d), dtype=np.float64)
    lse = np.zeros(cnt, dtype=np.float64)
    st = lib.oracle_attn_fwd(_ptr(q), _ptr(k), _ptr(v), n, d, float(scale), int(bool(causal)),
                             _iptr(r), cnt, _ptr(o), _ptr(lse), int(nthreads or default_threads()))
    if st != 0:
        raise RuntimeError(f"oracle_attn_fwd failed ({st})")
    return o, lse


def bwd(q, k, v, do, scale: float, causal: bool, qrows=None, krows=None,
        nthreads: int | None = None, lib=None):
    """Exact backward for one head.

    Returns ``(dQ[qrows], dK[krows], dV[krows], LSE, D)``; ``LSE`` and ``D``
    cover every row.  ``qrows``/``krows`` None means all rows.
    """
    lib = lib or load()
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(do)
    n, d = q.shape
    qr = None if qrows is None else np.ascontiguousarray(qrows, dtype=np.int64)
    kr = None if krows is None else np.ascontiguousarray(krows, dtype=np.int64)
    nq = n if qr is None else qr.shape[0]
    nk = n if kr is None else kr.shape[0]
    dq = np.zeros((nq, d)); dk = np.zeros((nk, d)); dv = np.zeros((nk, d))
    lse = np.zeros(n); dsum = np.zeros(n)
    st = lib.oracle_attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(do), n, d, float(scale), int(bool(causal)),
                             _iptr(qr), nq, _iptr(kr), nk, _ptr(dq), _ptr(dk), _ptr(dv),
                             _ptr(lse), _ptr(dsum), int(nthreads or default_threads()))
    if st != 0:
        raise RuntimeError(f"oracle_attn_bwd failed ({st})")
    return dq, dk, dv, lse, dsum


def fwd_all(Q, K, V, scale: float, causal: bool, nthreads: int | None = None):
    """Forward over a whole B x H x N x d batch (fp64 arrays): returns O, LSE."""
    B, H, N, d = Q.shape
    O = np.zeros((B, H, N, d)); L = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            O[b, h], L[b, h] = fwd(Q[b, h], K[b, h], V[b, h], scale, causal, nthreads=nthreads)
    return O, L


def bwd_all(Q, K, V, dO, scale: float, causal: bool, nthreads: int | None = None):
    """Backward over a whole B x H x N x d batch: returns dQ, dK, dV, LSE, D."""
    B, H, N, d = Q.shape
    dQ = np.zeros((B, H, N, d)); dK = np.zeros_like(dQ); dV = np.zeros_like(dQ)
    L = np.zeros((B, H, N)); Dd = np.zeros((B, H, N))
    for b in range(B):
        for h in range(H):
            dQ[b, h], dK[b, h], dV[b, h], L[b, h], Dd[b, h] = bwd(Q[b, h], K[b, h], V[b, h], dO[b, h],
                                                                  scale, causal, nthreads=nthreads)
    return dQ, dK, dV, L, Dd

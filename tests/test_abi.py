"""The C-ABI library: loads, exports every declared symbol, validates on the host (CPU only).

Only argument checks that return before any CUDA call are exercised here; no
kernel is launched.
"""
import ctypes
import os
import re

import pytest

from exact_attention_159_b200 import _lib, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _lib.lib()


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    assert declared_symbols() == sorted(_lib.SIGNATURES)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_no_torch_types_in_header():
    text = open(HEADER).read()
    assert "torch" not in text.lower().replace("pytorch", "")


def test_strerror_and_version(lib):
    for code in range(6):
        assert lib.fa_strerror(code)
    assert lib.fa_strerror(99) == b"unknown status"
    assert lib.fa_version() >= 100


P = ctypes.c_void_p(0x10000)   # fake, 16-byte aligned: never dereferenced by the checks below
P2 = ctypes.c_void_p(0x20000)
MIS = ctypes.c_void_p(0x10008)


def fwd(lib, q=P, k=P, v=P, o=P2, l=P2, B=1, H=1, N=128, d=64, scale=0.125, causal=0):
    return lib.fa_fwd(q, k, v, o, l, B, H, N, d, scale, causal, None)


def test_fwd_host_validation(lib):
    assert fwd(lib, d=96) == _lib.FA_ERR_UNSUPPORTED
    assert fwd(lib, d=256) == _lib.FA_ERR_UNSUPPORTED
    assert fwd(lib, B=-1) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, N=-5) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, causal=2) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, scale=0.0) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, scale=-1.0) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, scale=float("inf")) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, scale=float("nan")) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, q=None) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, l=None) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, k=MIS) == _lib.FA_ERR_ALIGNMENT
    # an empty problem is a no-op
    assert fwd(lib, B=0) == _lib.FA_OK
    assert fwd(lib, N=0) == _lib.FA_OK
    # output overlapping an input
    assert fwd(lib, o=P) == _lib.FA_ERR_INVALID_ARG
    assert fwd(lib, B=1 << 20, H=1 << 12) == _lib.FA_ERR_UNSUPPORTED


def test_bwd_host_validation(lib):
    ws = lib.fa_bwd_workspace_size(1, 1, 128, 64)
    base = dict(B=1, H=1, N=128, d=64)

    def bwd(ptrs=None, wsb=ws, scale=0.125, causal=0, **kw):
        a = dict(base, **kw)
        p = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(10)]
        if ptrs:
            for i, v in ptrs.items():
                p[i] = v
        return lib.fa_bwd(*p, wsb, a["B"], a["H"], a["N"], a["d"], scale, causal, None)

    assert bwd(d=80) == _lib.FA_ERR_UNSUPPORTED
    assert bwd(ptrs={9: None}) == _lib.FA_ERR_INVALID_ARG
    assert bwd(ptrs={5: MIS}) == _lib.FA_ERR_ALIGNMENT
    assert bwd(wsb=ws - 1) == _lib.FA_ERR_INVALID_ARG
    assert bwd(ptrs={6: ctypes.c_void_p(0x100000)}) == _lib.FA_ERR_INVALID_ARG   # dQ aliases Q
    assert bwd(ptrs={8: ctypes.c_void_p(0x800000)}) == _lib.FA_ERR_INVALID_ARG   # dV aliases dK
    assert bwd(B=0) == _lib.FA_OK


def test_workspace_size(lib):
    def expect(B, H, N, d):
        npad = (N + 127) // 128 * 128
        r = lambda x: (x + 255) // 256 * 256
        return r(B * H * npad * d * 4) + 2 * r(B * H * npad * 4)
    for shape in ((1, 1, 128, 64), (2, 3, 1000, 128), (1, 16, 32768, 128), (8, 16, 2048, 64), (1, 1, 1, 64)):
        assert lib.fa_bwd_workspace_size(*shape) == expect(*shape)
    assert lib.fa_bwd_workspace_size(0, 1, 128, 64) == 0
    assert lib.fa_bwd_workspace_size(1, 1, 128, 96) == 0


def test_softmax_options_validation(lib):
    assert lib.fa_set_softmax_options(-1.0, 1) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_set_softmax_options(8.0, 3) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_set_softmax_options(8.0, 8) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_set_softmax_options(8.0, -2) == _lib.FA_ERR_INVALID_ARG
    for share in (-1, 1, 2, 4):
        assert lib.fa_set_softmax_options(8.0, share) == _lib.FA_OK
    assert lib.fa_set_softmax_options(0.0, 0) == _lib.FA_OK
    assert lib.fa_set_softmax_options(8.0, -1) == _lib.FA_OK


def test_exp2_eval_validation(lib):
    assert lib.fa_exp2_eval(P, P2, 10, 3, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_exp2_eval(P, P2, 10, -1, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_exp2_eval(MIS, P2, 10, 0, None) == _lib.FA_ERR_ALIGNMENT
    assert lib.fa_exp2_eval(P, P2, 0, 0, None) == _lib.FA_OK


def test_profile_hook_validation(lib):
    assert lib.fa_profile_next(2, None, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_profile_next(0, P, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_profile_next(1, None, None) == _lib.FA_OK


def test_qk_host_validation(lib):
    p = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(10)]

    def fwd_qk(B=1, Hq=4, Hkv=2, Nq=128, Nk=256, d=64, scale=0.125, causal=1, ptrs=None):
        a = list(p[:5])
        for i, v in (ptrs or {}).items():
            a[i] = v
        return lib.fa_fwd_qk(*a, B, Hq, Hkv, Nq, Nk, d, scale, causal, None)

    assert fwd_qk(Hq=3, Hkv=2) == _lib.FA_ERR_INVALID_ARG      # Hq not a multiple of Hkv
    assert fwd_qk(Hkv=0) == _lib.FA_ERR_INVALID_ARG
    assert fwd_qk(Hkv=-1) == _lib.FA_ERR_INVALID_ARG
    assert fwd_qk(Nk=0) == _lib.FA_ERR_INVALID_ARG             # queries with no key set
    assert fwd_qk(Nk=-3) == _lib.FA_ERR_INVALID_ARG
    assert fwd_qk(d=96) == _lib.FA_ERR_UNSUPPORTED
    assert fwd_qk(ptrs={1: MIS}) == _lib.FA_ERR_ALIGNMENT
    assert fwd_qk(ptrs={3: p[1]}) == _lib.FA_ERR_INVALID_ARG   # O aliases K
    assert fwd_qk(Nq=0) == _lib.FA_OK and fwd_qk(B=0) == _lib.FA_OK and fwd_qk(Hq=0, Hkv=0) == _lib.FA_OK
    ws = lib.fa_bwd_qk_workspace_size(1, 4, 128, 64)
    assert ws == lib.fa_bwd_workspace_size(1, 4, 128, 64) > 0

    def bwd_qk(wsb=ws, Hq=4, Hkv=2, Nk=256, ptrs=None):
        a = list(p)
        for i, v in (ptrs or {}).items():
            a[i] = v
        return lib.fa_bwd_qk(*a, wsb, 1, Hq, Hkv, 128, Nk, 64, 0.125, 1, None)

    assert bwd_qk(Hq=4, Hkv=3) == _lib.FA_ERR_INVALID_ARG
    assert bwd_qk(wsb=ws - 1) == _lib.FA_ERR_INVALID_ARG
    assert bwd_qk(ptrs={7: ctypes.c_void_p(0x200000)}) == _lib.FA_ERR_INVALID_ARG   # dK aliases K
    assert bwd_qk(ptrs={8: MIS}) == _lib.FA_ERR_ALIGNMENT


def test_merge_helpers_host_validation(lib):
    A, A2, L1, L2 = (ctypes.c_void_p(0x100000 * i) for i in (1, 2, 3, 4))
    assert lib.fa_lse_merge(A, L1, A2, L2, 128, 96, 0, None) == _lib.FA_ERR_UNSUPPORTED
    assert lib.fa_lse_merge(A, L1, A2, L2, -1, 128, 0, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_lse_merge(A, L1, A2, L2, 128, 128, 2, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_lse_merge(None, L1, A2, L2, 128, 128, 0, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_lse_merge(MIS, L1, A2, L2, 128, 128, 0, None) == _lib.FA_ERR_ALIGNMENT
    assert lib.fa_lse_merge(A, L1, A, L2, 128, 128, 0, None) == _lib.FA_ERR_INVALID_ARG   # accumulator over the partial
    assert lib.fa_lse_merge(A, L1, A2, L2, 0, 128, 0, None) == _lib.FA_OK
    assert lib.fa_accumulate_bf16(A2, A, 12, 0, None) == _lib.FA_ERR_INVALID_ARG         # not a multiple of 8
    assert lib.fa_accumulate_bf16(A2, MIS, 16, 0, None) == _lib.FA_ERR_ALIGNMENT
    assert lib.fa_convert_f32_bf16(A, A, 16, None) == _lib.FA_ERR_INVALID_ARG            # overlap
    assert lib.fa_convert_f32_bf16(A, A2, 0, None) == _lib.FA_OK


def test_variant_and_probe_host_validation(lib):
    assert lib.fa_set_backward_variant(2) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_set_backward_variant(-1) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_sm_clock_probe(None, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_sm_clock_probe(ctypes.c_void_p(0x100004), None) == _lib.FA_ERR_ALIGNMENT


def test_accumulating_forward_and_backward_pieces_host_validation(lib):
    A = [ctypes.c_void_p(0x100000 * (i + 1)) for i in range(8)]
    ws = lib.fa_bwd_qk_workspace_size(1, 2, 256, 64)

    def facc(q=A[0], k=A[1], v=A[2], o=A[3], l=A[4], first=1, d=64, causal=0, Hkv=2):
        return lib.fa_fwd_accumulate(q, k, v, o, l, 1, 2, Hkv, 256, 256, d, 0.125, causal, first, None)

    assert facc(first=2) == _lib.FA_ERR_INVALID_ARG
    assert facc(o=None) == _lib.FA_ERR_INVALID_ARG
    assert facc(l=MIS) == _lib.FA_ERR_ALIGNMENT
    assert facc(d=96) == _lib.FA_ERR_UNSUPPORTED
    assert facc(Hkv=3) == _lib.FA_ERR_INVALID_ARG                  # Hq not a multiple of Hkv
    assert facc(o=ctypes.c_void_p(0x100000)) == _lib.FA_ERR_INVALID_ARG   # O_acc aliases Q

    def prep(o=A[0], do=A[1], l=A[2], w=A[3], wsb=ws):
        return lib.fa_bwd_prepare(o, do, l, w, wsb, 1, 2, 256, 64, None)

    assert prep(w=None) == _lib.FA_ERR_INVALID_ARG
    assert prep(wsb=ws - 1) == _lib.FA_ERR_INVALID_ARG
    assert prep(do=MIS) == _lib.FA_ERR_ALIGNMENT
    assert prep(w=ctypes.c_void_p(0x100000)) == _lib.FA_ERR_INVALID_ARG  # workspace aliases O

    def acc(q=A[0], k=A[1], v=A[2], do=A[3], w=A[4], dk=A[5], dv=A[6], first=0, wsb=ws):
        return lib.fa_bwd_accumulate(q, k, v, do, w, wsb, dk, dv, 1, 2, 2, 256, 256, 64, 0.125, 1, first, None)

    assert acc(first=-1) == _lib.FA_ERR_INVALID_ARG
    assert acc(dk=None) == _lib.FA_ERR_INVALID_ARG
    assert acc(dv=MIS) == _lib.FA_ERR_ALIGNMENT
    assert acc(wsb=16) == _lib.FA_ERR_INVALID_ARG
    assert acc(dk=ctypes.c_void_p(0x700000)) == _lib.FA_ERR_INVALID_ARG  # dK_acc aliases dV_acc

    assert lib.fa_bwd_finish(None, ws, A[0], 1, 2, 256, 64, 0.125, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_finish(A[1], ws - 16, A[0], 1, 2, 256, 64, 0.125, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_finish(A[1], ws, A[1], 1, 2, 256, 64, 0.125, None) == _lib.FA_ERR_INVALID_ARG
    assert lib.fa_bwd_finish(A[1], ws, A[0], 0, 2, 256, 64, 0.125, None) == _lib.FA_OK  # empty

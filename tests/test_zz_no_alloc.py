"""fa_bwd_noalloc: the backward pass for callers that cannot allocate device
memory (for example a process whose memory manager already owns the whole
GPU, or latency-critical code that must not trigger cudaMalloc's implicit
synchronisation).  It runs on a fixed scratch array inside the library
instead of a caller workspace.

Checked here through the C ABI: two calls in a row each match the existing
fa_bwd entry point within the gradient tolerance the parity tests use, and a
problem too large for the scratch array is refused before anything runs.
This file is collected last so that a stop-at-first-failure run has already
run every other test when it gets here.
"""
import ctypes

import pytest
import torch

from exact_attention_159_b200 import _lib, api, build
from tests.gpu_util import TOL_GRAD, Case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    yield
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == (0, 0)


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _rel(a, b):
    a, b = a.double(), b.double()
    return float((a - b).norm() / b.norm())


# the last case fills the scratch array to within 16 KB: 16 x 8064 = 129,024 rows at d = 128
@pytest.mark.parametrize("B,H,N,d,causal", [(1, 4, 1000, 128, True), (2, 3, 640, 64, False),
                                            (1, 16, 8064, 128, True)])
def test_noalloc_matches_fa_bwd_twice(B, H, N, d, causal):
    c = Case(B, H, N, d, causal, seed_workload=21, bwd=True)
    o, lse = c.fwd_gpu()
    ref = c.bwd_gpu(o, lse)                       # existing entry point, caller workspace
    lib = _lib.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):                         # the scratch keeps the previous call's contents
        dq, dk, dv = (torch.full_like(c.dev["q"], float("nan")) for _ in range(3))
        rc = lib.fa_bwd_noalloc(_p(c.dev["q"]), _p(c.dev["k"]), _p(c.dev["v"]), _p(o), _p(c.dev["do"]), _p(lse),
                                _p(dq), _p(dk), _p(dv), B, H, N, d, c.scale, int(causal), stream)
        assert rc == 0, lib.fa_strerror(rc)
        torch.cuda.synchronize()
        for got, want, name in ((dq, ref[0], "dQ"), (dk, ref[1], "dK"), (dv, ref[2], "dV")):
            assert torch.isfinite(got.float()).all(), f"call {call}: {name} not fully written"
            assert _rel(got, want) <= TOL_GRAD, f"call {call}: {name} differs from fa_bwd"


def test_noalloc_refuses_problems_beyond_the_scratch():
    lib = _lib.lib()
    fake = ctypes.c_void_p(0x100000)
    # B=1, H=16, N=32768, d=128 needs 272 MB of workspace: refused on the host, nothing launched
    rc = lib.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, 1, 16, 32768, 128, 0.088, 1, None)
    assert rc == _lib.FA_ERR_UNSUPPORTED


def test_noalloc_limit_is_exact():
    lib = _lib.lib()
    limit = 64 << 20  # FA_BWD_NOALLOC_SCRATCH_BYTES in include/fa.h
    # the largest problem at d = 128 fits, one more 128-row tile does not
    assert lib.fa_bwd_workspace_size(1, 16, 8064, 128) <= limit
    assert lib.fa_bwd_workspace_size(1, 1, 129024 + 128, 128) > limit
    fake = ctypes.c_void_p(0x100000)
    for shape in ((1, 1, 129024 + 128, 128), (1, 16, 8065, 128), (1, 2, 254080 // 2 + 128, 64)):
        rc = lib.fa_bwd_noalloc(fake, fake, fake, fake, fake, fake, fake, fake, fake, *shape, 0.088, 1, None)
        assert rc == _lib.FA_ERR_UNSUPPORTED, shape

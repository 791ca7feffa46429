"""Failure detection on the GPU without a fault: a kernel whose pipeline wait
can never complete must give up after its bounded wait and report
FA_ERR_TIMEOUT through the status word; the context stays usable."""
import ctypes

import pytest
import torch

from exact_attention_159_b200 import _lib, api, build
from tests.gpu_util import Case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def test_bounded_wait_reports_timeout_and_context_survives():
    lib = _lib.lib()
    assert api.fa_last_device_status() == (0, 0)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert lib.fa_selftest_wait_timeout(stream) == _lib.FA_OK
    rc, detail = api.fa_last_device_status()
    assert rc == _lib.FA_ERR_TIMEOUT and detail == 0xF01
    # the status is cleared and the device still runs the real kernels correctly
    assert api.fa_last_device_status() == (0, 0)
    c = Case(1, 1, 256, 64, True, seed_workload=31)
    o, lse = c.fwd_gpu()
    o_ref, l_ref = c.oracle_fwd(0, 0)
    from tests.gpu_util import bf16_to_f64
    assert abs(bf16_to_f64(o)[0, 0] - o_ref).max() <= 1e-2
    assert api.fa_last_device_status() == (0, 0)

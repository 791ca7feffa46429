"""The SM clock probe returns the clock the device is running at (within the B200's range)."""
import pytest
import torch

from exact_attention_159_b200 import api, build

pytestmark = pytest.mark.gpu


def test_sm_clock_probe_is_plausible():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    mhz = [api.fa_sm_clock_probe() for _ in range(3)]
    assert all(300.0 < m < 2500.0 for m in mhz), mhz
    assert api.fa_last_device_status() == (0, 0)

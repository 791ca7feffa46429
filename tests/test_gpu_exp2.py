"""Device exp2: the cubic software path matches its host emulation bit for bit
and fp64 exp2 within 2e-4 relative over [-126, 0]; the SFU path too."""
import numpy as np
import pytest
import torch

from exact_attention_159_b200 import api, build
from tests.exp2_host import exp2_poly_f32, sweep_points

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()


def test_poly_matches_host_emulation_and_fp64():
    x = sweep_points()
    y = api.fa_exp2_eval(torch.from_numpy(x).cuda(), mode=0).cpu().numpy()
    host = exp2_poly_f32(x)
    ulps = np.abs(y.view(np.int32).astype(np.int64) - host.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1, ulps.max()
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    print(f"poly exp2: max rel err {rel.max():.3e} over {x.size} points; host/device max ulp {ulps.max()}")
    assert rel.max() <= 2e-4


def test_sfu_exp2_and_masked_input():
    x = sweep_points(1 << 20)
    y = api.fa_exp2_eval(torch.from_numpy(x).cuda(), mode=1).cpu().numpy()
    rel = np.abs(y.astype(np.float64) / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() <= 1e-6
    z = api.fa_exp2_eval(torch.tensor([-np.inf, 0.0, 8.0, -200.0], dtype=torch.float32, device="cuda"), mode=1)
    assert z.cpu().tolist() == [0.0, 1.0, 256.0, 0.0]


def test_packed_poly_equals_scalar_poly():
    x = sweep_points(1 << 22)
    xd = torch.from_numpy(x).cuda()
    a = api.fa_exp2_eval(xd, mode=0).cpu().numpy()
    b = api.fa_exp2_eval(xd, mode=2).cpu().numpy()
    assert np.array_equal(a.view(np.int32), b.view(np.int32))

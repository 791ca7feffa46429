"""The forward and backward captured in a CUDA graph and replayed: the library makes no
allocation and no synchronising call inside a launch, so a captured step replays with the
results of eager calls."""
import pytest
import torch

from exact_attention_159_b200 import api, build
from tests.gpu_util import Case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    yield
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == (0, 0)


@pytest.mark.parametrize("d", [64, 128])
def test_fwd_bwd_replay_in_cuda_graph(d):
    c = Case(1, 4, 1024, d, True, seed_workload=15, bwd=True)
    q, k, v, do = (c.dev[x] for x in ("q", "k", "v", "do"))
    o_ref, l_ref = api.fa_fwd(q, k, v, c.scale, True)
    g_ref = api.fa_bwd(q, k, v, o_ref, do, l_ref, c.scale, True)
    o, lse = torch.empty_like(o_ref), torch.empty_like(l_ref)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(api.fa_bwd_workspace_size(1, 4, 1024, d), dtype=torch.uint8, device="cuda")
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):  # warm-up on the capture stream, as torch recommends
        api.fa_fwd(q, k, v, c.scale, True, out=o, lse=lse)
        api.fa_bwd(q, k, v, o, do, lse, c.scale, True, dq=dq, dk=dk, dv=dv, workspace=ws)
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        api.fa_fwd(q, k, v, c.scale, True, out=o, lse=lse)
        api.fa_bwd(q, k, v, o, do, lse, c.scale, True, dq=dq, dk=dk, dv=dv, workspace=ws)
    for x in (o, lse, dq, dk, dv):
        x.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    assert torch.equal(dk, g_ref[1]) and torch.equal(dv, g_ref[2])
    # dQ accumulates with fp32 reductions whose order varies: equal up to one bf16 ulp
    assert float((dq.float() - g_ref[0].float()).abs().max()) <= 2.0 ** -6 * float(g_ref[0].float().abs().max())

"""The Python binding refuses what the kernels cannot take, on the host, before any launch: in
particular CPU tensors raise instead of being computed some other way (there is no fallback)."""
import pytest
import torch

from exact_attention_159_b200 import api, build


@pytest.fixture(scope="module", autouse=True)
def _lib():
    build.build()


def _bf16(*shape):
    return torch.zeros(shape, dtype=torch.bfloat16)


def test_cpu_tensors_are_refused_not_computed():
    q = _bf16(1, 2, 64, 64)
    with pytest.raises(ValueError, match="CUDA"):
        api.fa_fwd(q, q.clone(), q.clone())
    lse = torch.zeros((1, 2, 64), dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA"):
        api.fa_bwd(q, q.clone(), q.clone(), q.clone(), q.clone(), lse)
    with pytest.raises(ValueError, match="CUDA"):
        api.fa_bwd_noalloc(q, q.clone(), q.clone(), q.clone(), q.clone(), lse)
    with pytest.raises(ValueError):
        api.fa_fwd_qk(q, _bf16(1, 1, 80, 64), _bf16(1, 1, 80, 64))


def test_wrong_dtype_shape_and_layout_are_refused():
    q = torch.zeros((1, 2, 64, 64), dtype=torch.float32)
    with pytest.raises(ValueError):
        api.fa_fwd(q, q.clone(), q.clone())
    with pytest.raises(ValueError):
        api.fa_fwd(_bf16(2, 64, 64), _bf16(2, 64, 64), _bf16(2, 64, 64))    # not [B, H, N, d]
    q = _bf16(1, 2, 64, 64)
    with pytest.raises(ValueError):
        api.fa_fwd(q, _bf16(1, 2, 32, 64), q.clone())                       # K of another length
    with pytest.raises(ValueError):
        api.fa_fwd(q.transpose(2, 3), q.clone(), q.clone())                  # not contiguous


def test_diagnostic_helpers_refuse_cpu_buffers():
    with pytest.raises(ValueError):
        api.fa_sm_clock_probe(torch.zeros(2, dtype=torch.int64))
    with pytest.raises(ValueError):
        api.fa_exp2_eval(torch.zeros(16, dtype=torch.float32))


def test_workspace_must_be_a_device_buffer_of_the_needed_size():
    from exact_attention_159_b200.api import _need_workspace
    with pytest.raises(ValueError, match="CUDA"):
        _need_workspace(torch.zeros(1 << 20, dtype=torch.uint8), 1024)   # host memory never reaches a kernel

"""GPU parity of the ring (context-parallel) pieces: the log-sum-exp merge, the fp32 helpers,
and the whole ring forward / backward for R ranks emulated in one process on one GPU (the
same per-rank steps as the distributed driver; the chunks are handed over in Python)."""
import math

import numpy as np
import pytest
import torch

from exact_attention_159_b200 import api, build, ring
from exact_attention_159_b200 import inputs as I
from oracle import oracle as OR
from tests.gpu_util import TOL_GRAD, TOL_LSE, TOL_O, bf16_to_f64, rel_l2, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    yield
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == (0, 0)


def _seq(seed, B, H, N, d):
    bits = I.attention_inputs(seed, B, H, N, d, with_do=True)
    return {k: to_dev(v) for k, v in bits.items()}, {k: I.bf16_bits_to_f64(v) for k, v in bits.items()}


@pytest.mark.parametrize("d", [64, 128])
def test_merge_of_two_key_halves_is_full_attention(d):
    B, H, Nq, Nk = 1, 4, 384, 1000
    dev, f64 = _seq(31, B, H, max(Nq, Nk), d)
    q = dev["q"][:, :, :Nq].contiguous()
    k, v = dev["k"][:, :, :Nk].contiguous(), dev["v"][:, :, :Nk].contiguous()
    scale = 1.0 / math.sqrt(d)
    half = 448
    o_a, l_a = api.fa_fwd_qk(q, k[:, :, :half].contiguous(), v[:, :, :half].contiguous(), scale, False)
    o_b, l_b = api.fa_fwd_qk(q, k[:, :, half:].contiguous(), v[:, :, half:].contiguous(), scale, False)
    o_acc = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    l_acc = torch.empty(q.shape[:-1], dtype=torch.float32, device="cuda")
    api.fa_lse_merge(o_a, l_a, o_acc, l_acc, first=True)
    api.fa_lse_merge(o_b, l_b, o_acc, l_acc)
    O = o_acc.double().cpu().numpy()
    L = l_acc.double().cpu().numpy()
    for h in range(H):
        o_ref, l_ref = OR.fwd(f64["q"][0, h, :Nq], f64["k"][0, h, :Nk], f64["v"][0, h, :Nk], scale, False)
        assert np.abs(O[0, h] - o_ref).max() <= TOL_O
        assert np.abs(L[0, h] - l_ref).max() <= TOL_LSE


def test_merge_with_rows_that_see_no_key():
    # causal with Nq > Nk: the first Nq - Nk rows have LSE = -inf in the partial
    B, H, Nq, Nk, d = 1, 2, 300, 200, 128
    dev, f64 = _seq(32, B, H, Nq, d)
    q, k, v = dev["q"], dev["k"][:, :, :Nk].contiguous(), dev["v"][:, :, :Nk].contiguous()
    o_p, l_p = api.fa_fwd_qk(q, k, v, None, True)
    o_acc = torch.empty(q.shape, dtype=torch.float32, device="cuda")
    l_acc = torch.empty(q.shape[:-1], dtype=torch.float32, device="cuda")
    api.fa_lse_merge(o_p, l_p, o_acc, l_acc, first=True)
    api.fa_lse_merge(o_p, l_p, o_acc, l_acc)  # the same keys twice: O unchanged, LSE + ln 2
    L = l_acc.double().cpu().numpy()
    Lp = l_p.double().cpu().numpy()
    blind = Nq - Nk
    assert np.all(np.isneginf(L[:, :, :blind])) and np.all(o_acc[:, :, :blind].cpu().numpy() == 0.0)
    np.testing.assert_allclose(L[:, :, blind:], Lp[:, :, blind:] + math.log(2.0), atol=1e-5)
    np.testing.assert_allclose(o_acc[:, :, blind:].cpu().numpy(), o_p[:, :, blind:].float().cpu().numpy(), atol=1e-6)


def test_accumulate_and_convert():
    x = torch.randn(4096, device="cuda").to(torch.bfloat16)
    y = torch.randn(4096, device="cuda").to(torch.bfloat16)
    acc = torch.empty(4096, dtype=torch.float32, device="cuda")
    api.fa_accumulate_bf16(acc, x, first=True)
    api.fa_accumulate_bf16(acc, y)
    assert torch.equal(acc, x.float() + y.float())
    out = api.fa_convert_f32_bf16(acc)
    assert torch.equal(out, acc.to(torch.bfloat16))


@pytest.mark.parametrize("world,causal", [(2, True), (4, True), (4, False)])
def test_emulated_ring_matches_oracle(world, causal):
    B, H, n, d = 1, 4, 512, 128
    N = n * world
    dev, f64 = _seq(33, B, H, N, d)
    scale = 1.0 / math.sqrt(d)
    ch = {k: [t[:, :, r * n:(r + 1) * n].contiguous() for r in range(world)] for k, t in dev.items()}
    os_, lses = ring.ring_attention_fwd_emulated(ch["q"], ch["k"], ch["v"], scale, causal)
    dqs, dks, dvs = ring.ring_attention_bwd_emulated(ch["q"], ch["k"], ch["v"], os_, ch["do"], lses, scale, causal)
    O = np.concatenate([bf16_to_f64(o) for o in os_], axis=2)
    L = np.concatenate([l.double().cpu().numpy() for l in lses], axis=2)
    dQ, dK, dV = (np.concatenate([bf16_to_f64(t) for t in ts], axis=2) for ts in (dqs, dks, dvs))
    worst = dict(O=0.0, LSE=0.0, dQ=0.0, dK=0.0, dV=0.0)
    for h in range(H):
        qr, kr = sample_rows(N, 96, h), sample_rows(N, 96, h + 50)
        o_ref, l_ref = OR.fwd(f64["q"][0, h], f64["k"][0, h], f64["v"][0, h], scale, causal, rows=qr)
        dq_ref, dk_ref, dv_ref, _, _ = OR.bwd(f64["q"][0, h], f64["k"][0, h], f64["v"][0, h], f64["do"][0, h], scale,
                                              causal, qrows=qr, krows=kr)
        worst["O"] = max(worst["O"], float(np.abs(O[0, h][qr] - o_ref).max()))
        worst["LSE"] = max(worst["LSE"], float(np.abs(L[0, h][qr] - l_ref).max()))
        worst["dQ"] = max(worst["dQ"], rel_l2(dQ[0, h][qr], dq_ref))
        worst["dK"] = max(worst["dK"], rel_l2(dK[0, h][kr], dk_ref))
        worst["dV"] = max(worst["dV"], rel_l2(dV[0, h][kr], dv_ref))
    print(f"[ring world {world} causal {causal}] " + "  ".join(f"{k} {v:.3e}" for k, v in worst.items()))
    assert worst["O"] <= TOL_O and worst["LSE"] <= TOL_LSE
    assert worst["dQ"] <= TOL_GRAD and worst["dK"] <= TOL_GRAD and worst["dV"] <= TOL_GRAD

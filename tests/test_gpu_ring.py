"""GPU parity of the ring (context-parallel) pieces: the log-sum-exp merge, the accumulating
forward and backward entry points over several key blocks, the fp32 helpers, and the whole
ring forward / backward (zig-zag layout) for R ranks emulated in one process on one GPU (the
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


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_accumulating_calls_over_key_blocks_equal_full_attention(d, causal):
    # fa_fwd_accumulate / fa_bwd_accumulate over three key blocks (the causal square last, so the
    # earlier blocks are entirely visible) against the oracle on the whole key set
    B, H, Nq = 1, 3, 384
    blocks = [256, 384, 384]  # the last block holds the queries' own keys
    Nk = sum(blocks)
    dev, f64 = _seq(34, B, H, Nk, d)
    q, do = dev["q"][:, :, Nk - Nq:].contiguous(), dev["do"][:, :, Nk - Nq:].contiguous()
    scale = 1.0 / math.sqrt(d)
    o_acc = torch.full(q.shape, float("nan"), dtype=torch.float32, device="cuda")
    l_acc = torch.full(q.shape[:-1], float("nan"), dtype=torch.float32, device="cuda")
    starts = np.cumsum([0] + blocks[:-1])
    kb = [(dev["k"][:, :, s:s + n].contiguous(), dev["v"][:, :, s:s + n].contiguous()) for s, n in zip(starts, blocks)]
    for i, (k, v) in enumerate(kb):
        last = i == len(kb) - 1
        api.fa_fwd_accumulate(q, k, v, o_acc, l_acc, scale, causal and last, first=(i == 0))
    o = api.fa_convert_f32_bf16(o_acc)
    ws = api.fa_bwd_prepare(o, do, l_acc)
    dk_acc = [torch.full(k.shape, float("nan"), dtype=torch.float32, device="cuda") for k, _ in kb]
    dv_acc = [torch.full(k.shape, float("nan"), dtype=torch.float32, device="cuda") for k, _ in kb]
    for i, (k, v) in enumerate(kb):
        last = i == len(kb) - 1
        api.fa_bwd_accumulate(q, k, v, do, ws, dk_acc[i], dv_acc[i], scale, causal and last, first=True)
        api.fa_bwd_accumulate(q, k, v, do, ws, dk_acc[i], dv_acc[i], scale, causal and last, first=False)
    dq = api.fa_bwd_finish(ws, B, H, Nq, d, scale)
    # every block ran twice in the backward: dQ, dK and dV are twice the gradients
    O, L = o_acc.double().cpu().numpy(), l_acc.double().cpu().numpy()
    dQ = bf16_to_f64(dq) / 2.0
    dK = np.concatenate([a.double().cpu().numpy() for a in dk_acc], axis=2) / 2.0
    dV = np.concatenate([a.double().cpu().numpy() for a in dv_acc], axis=2) / 2.0
    for h in range(H):
        x = {k: f64[k][0, h] for k in f64}
        o_ref, l_ref = OR.fwd(x["q"][Nk - Nq:], x["k"], x["v"], scale, causal)
        dq_ref, dk_ref, dv_ref, _, _ = OR.bwd(x["q"][Nk - Nq:], x["k"], x["v"], x["do"][Nk - Nq:], scale, causal)
        assert np.abs(O[0, h] - o_ref).max() <= TOL_O
        assert np.abs(L[0, h] - l_ref).max() <= TOL_LSE
        assert rel_l2(dQ[0, h], dq_ref) <= TOL_GRAD
        assert rel_l2(dK[0, h], dk_ref) <= TOL_GRAD
        assert rel_l2(dV[0, h], dv_ref) <= TOL_GRAD


def test_accumulate_f32():
    x = torch.randn(4096, device="cuda")
    acc = torch.randn(4096, device="cuda")
    want = acc + x
    api.fa_accumulate_f32(acc, x)
    assert torch.equal(acc, want)


@pytest.mark.parametrize("world,causal", [(2, True), (4, True), (4, False), (3, True)])
def test_emulated_ring_matches_oracle(world, causal):
    B, H, n, d = 1, 4, 512, 128
    N = n * world
    dev, f64 = _seq(33, B, H, N, d)
    scale = 1.0 / math.sqrt(d)
    ch = {k: [ring.zigzag_shard(t, r, world) for r in range(world)] for k, t in dev.items()}
    os_, lses = ring.ring_attention_fwd_emulated(ch["q"], ch["k"], ch["v"], scale, causal)
    dqs, dks, dvs = ring.ring_attention_bwd_emulated(ch["q"], ch["k"], ch["v"], os_, ch["do"], lses, scale, causal)
    O = bf16_to_f64(ring.zigzag_unshard(os_))
    L = ring.zigzag_unshard(lses).double().cpu().numpy()
    dQ, dK, dV = (bf16_to_f64(ring.zigzag_unshard(ts)) for ts in (dqs, dks, dvs))
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

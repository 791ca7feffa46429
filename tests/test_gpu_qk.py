"""GPU parity of grouped-query attention (Hq query heads over Hkv key/value heads) and of
unequal query / key lengths (causal aligned at the last query and key), through the C ABI
(fa_fwd_qk / fa_bwd_qk), against the fp64 oracle on the same seeded bf16 inputs."""
import math

import numpy as np
import pytest
import torch

from exact_attention_159_b200 import api, build
from exact_attention_159_b200 import inputs as I
from oracle import oracle as OR
from tests.gpu_util import TOL_GRAD, TOL_LSE, TOL_O, bf16_to_f64, rel_l2, sample_rows, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    build.build()
    api.fa_set_softmax_options(8.0, -1)
    yield
    torch.cuda.synchronize()
    assert api.fa_last_device_status() == (0, 0)


class QKCase:
    def __init__(self, B, Hq, Hkv, Nq, Nk, d, causal, seed):
        self.B, self.Hq, self.Hkv, self.Nq, self.Nk, self.d, self.causal = B, Hq, Hkv, Nq, Nk, d, causal
        self.G = Hq // Hkv
        self.scale = 1.0 / math.sqrt(d)
        self.bits = I.attention_inputs_qk(seed, B, Hq, Hkv, Nq, Nk, d, with_do=True)
        self.dev = {k: to_dev(v) for k, v in self.bits.items()}
        self.f64 = {k: I.bf16_bits_to_f64(v) for k, v in self.bits.items()}

    def gpu(self):
        o, lse = api.fa_fwd_qk(self.dev["q"], self.dev["k"], self.dev["v"], self.scale, self.causal)
        grads = api.fa_bwd_qk(self.dev["q"], self.dev["k"], self.dev["v"], o, self.dev["do"], lse, self.scale,
                              self.causal)
        return o, lse, grads


def seen_rows(c, rows):
    """Query rows that see at least one key."""
    rows = np.asarray(rows)
    return rows[rows + (c.Nk - c.Nq) >= 0] if c.causal else rows


def check(c, q_rows_per_head=None, k_rows_per_head=None, label="", o_rel=0.0):
    """Compare with the oracle; an O element may differ by TOL_O + o_rel * |O_ref| (o_rel = 2^-8 covers
    the bf16 rounding of the output, half an ulp, which alone exceeds TOL_O once |O_ref| >= 4)."""
    o, lse, (dq, dk, dv) = c.gpu()
    O, L = bf16_to_f64(o), lse.cpu().numpy().astype(np.float64)
    dQ, dK, dV = bf16_to_f64(dq), bf16_to_f64(dk), bf16_to_f64(dv)
    worst = dict(O=0.0, LSE=0.0, dQ=0.0, dK=0.0, dV=0.0)
    for b in range(c.B):
        qr = None if q_rows_per_head is None else sample_rows(c.Nq, q_rows_per_head, 7 * b + 1)
        kr = None if k_rows_per_head is None else sample_rows(c.Nk, k_rows_per_head, 7 * b + 2)
        Q, K, V, dO = (c.f64[x][b] for x in ("q", "k", "v", "do"))
        o_ref, l_ref = OR.gqa_fwd(Q, K, V, c.scale, c.causal, rows=qr)
        dq_ref, dk_ref, dv_ref, _, _ = OR.gqa_bwd(Q, K, V, dO, c.scale, c.causal, qrows=qr, krows=kr)
        qs = np.arange(c.Nq) if qr is None else qr
        ks = np.arange(c.Nk) if kr is None else kr
        vis = np.isin(qs, seen_rows(c, qs))
        for h in range(c.Hq):
            worst["O"] = max(worst["O"], float((np.abs(O[b, h][qs] - o_ref[h]) - o_rel * np.abs(o_ref[h])).max()))
            if vis.any():
                worst["LSE"] = max(worst["LSE"], float(np.abs(L[b, h][qs][vis] - l_ref[h][vis]).max()))
            if (~vis).any():  # rows that see no key
                assert np.all(np.isneginf(L[b, h][qs][~vis])), f"{label}: LSE of a row with no key"
                assert np.all(O[b, h][qs][~vis] == 0.0) and np.all(dQ[b, h][qs][~vis] == 0.0)
            worst["dQ"] = max(worst["dQ"], rel_l2(dQ[b, h][qs], dq_ref[h]))
        for g in range(c.Hkv):
            worst["dK"] = max(worst["dK"], rel_l2(dK[b, g][ks], dk_ref[g]))
            worst["dV"] = max(worst["dV"], rel_l2(dV[b, g][ks], dv_ref[g]))
    print(f"[{label}] " + "  ".join(f"{k} {v:.3e}" for k, v in worst.items()))
    assert worst["O"] <= TOL_O and worst["LSE"] <= TOL_LSE, (label, worst)
    for k in ("dQ", "dK", "dV"):
        assert worst[k] <= TOL_GRAD, (label, k, worst[k])


SMALL = [  # B, Hq, Hkv, Nq, Nk, d, causal
    (2, 4, 2, 256, 256, 128, True), (2, 4, 2, 256, 256, 128, False), (1, 6, 1, 200, 200, 64, True),
    (1, 2, 2, 256, 1000, 128, True), (1, 2, 2, 256, 1000, 128, False), (1, 2, 2, 1000, 256, 128, True),
    (1, 2, 2, 1000, 256, 64, False), (1, 4, 2, 200, 383, 128, True), (1, 2, 1, 1, 513, 128, True),
    (1, 2, 1, 383, 129, 64, True), (2, 4, 4, 640, 640, 64, True), (1, 8, 2, 384, 2048, 128, True),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", SMALL,
                         ids=[f"B{b}-H{hq}/{hk}-{nq}x{nk}-d{d}-{'c' if c else 'f'}" for b, hq, hk, nq, nk, d, c in SMALL])
def test_qk_full(B, Hq, Hkv, Nq, Nk, d, causal):
    c = QKCase(B, Hq, Hkv, Nq, Nk, d, causal, seed=21)
    check(c, label=f"B{B} H{Hq}/{Hkv} {Nq}x{Nk} d{d} c{int(causal)}")


def test_qk_prefill_against_cache_large():
    # 2048 new queries over an 8192-key cache, 32 query heads on 8 key/value heads
    c = QKCase(1, 32, 8, 2048, 8192, 128, True, seed=22)
    check(c, q_rows_per_head=48, k_rows_per_head=48, label="prefill 2048 over 8192, H 32/8")


def test_qk_square_matches_fa_fwd():
    c = QKCase(1, 4, 4, 640, 640, 128, True, seed=23)
    o1, l1 = api.fa_fwd(c.dev["q"], c.dev["k"], c.dev["v"], c.scale, True)
    o2, l2 = api.fa_fwd_qk(c.dev["q"], c.dev["k"], c.dev["v"], c.scale, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_gqa_equals_repeated_heads():
    # the grouped call against plain attention with each key/value head repeated for its group
    c = QKCase(1, 8, 2, 512, 512, 128, True, seed=24)
    o, lse = api.fa_fwd_qk(c.dev["q"], c.dev["k"], c.dev["v"], c.scale, True)
    kr = c.dev["k"].repeat_interleave(c.G, dim=1).contiguous()
    vr = c.dev["v"].repeat_interleave(c.G, dim=1).contiguous()
    o2, l2 = api.fa_fwd(c.dev["q"], kr, vr, c.scale, True)
    assert torch.equal(o, o2) and torch.equal(lse, l2)


@pytest.mark.parametrize("Hq,Hkv,Nq,Nk,d", [(4, 2, 300, 300, 128), (2, 2, 200, 456, 128), (2, 2, 300, 300, 64)],
                         ids=["gqa", "nq-ne-nk", "d64"])
def test_backward_pair_switch_leaves_other_shapes_to_the_single_cta_kernel(Hq, Hkv, Nq, Nk, d):
    # the cluster-pair backward covers d = 128, Hq == Hkv, Nq == Nk only; with it selected, every
    # other shape still runs (and equals) the single-CTA kernel
    c = QKCase(1, Hq, Hkv, Nq, Nk, d, True, seed=61)
    o, lse = api.fa_fwd_qk(c.dev["q"], c.dev["k"], c.dev["v"], c.scale, True)
    g0 = api.fa_bwd_qk(c.dev["q"], c.dev["k"], c.dev["v"], o, c.dev["do"], lse, c.scale, True)
    api.fa_set_backward_variant(1)
    try:
        g1 = api.fa_bwd_qk(c.dev["q"], c.dev["k"], c.dev["v"], o, c.dev["do"], lse, c.scale, True)
    finally:
        api.fa_set_backward_variant(0)
    assert torch.equal(g0[1], g1[1]) and torch.equal(g0[2], g1[2])   # dK, dV: same kernel, same bits
    assert float((g0[0].float() - g1[0].float()).abs().max()) <= 2.0 ** -6 * float(g0[0].float().abs().max())


# Many more work units than SMs, so every persistent forward CTA walks several units: an odd number
# of query tiles (the second tile of every other unit is absent), query tiles that see no key
# (causal with Nq > Nk), and grouped heads.  All rows of every head are compared with the oracle.
# With this many rows, early causal rows (one or two visible keys) reach |O| >= 4, where rounding O
# to bf16 alone costs up to 0.0156, so the O bound adds that half-ulp: TOL_O + 2^-8 |O_ref|.
MANY_UNITS = [  # B, Hq, Hkv, Nq, Nk, d, causal
    (1, 320, 320, 383, 383, 128, True), (1, 320, 40, 1000, 256, 64, True), (2, 160, 160, 200, 200, 64, False),
    (1, 300, 100, 640, 640, 128, False),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nq,Nk,d,causal", MANY_UNITS,
                         ids=[f"B{b}-H{hq}x{hk}-{nq}x{nk}-d{d}-{'c' if c else 'f'}"
                              for b, hq, hk, nq, nk, d, c in MANY_UNITS])
def test_persistent_forward_many_units_per_cta(B, Hq, Hkv, Nq, Nk, d, causal):
    check(QKCase(B, Hq, Hkv, Nq, Nk, d, causal, seed=77), label=f"units B{B} H{Hq}/{Hkv} {Nq}x{Nk} d{d}",
          o_rel=2.0 ** -8)

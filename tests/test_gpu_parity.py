"""GPU parity: libfa (through the C ABI) against the fp64 oracle on identical
seeded bf16 inputs.

Small shapes are compared element by element in full; the full-size workloads
are compared on sampled rows (each query row of O / LSE / dQ, and each key row
of dK / dV, is computable by the oracle on its own), plus invariants that hold
at any size.
"""
import numpy as np
import pytest
import torch

from exact_attention_159_b200 import _lib, api, build
from tests.gpu_util import TOL_GRAD, TOL_LSE, TOL_O, Case, bf16_to_f64, rel_l2, sample_rows

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


def check_fwd(case, o, lse, heads, rows_per_head, label):
    O_gpu = bf16_to_f64(o)
    L_gpu = lse.cpu().numpy().astype(np.float64)
    worst_o = worst_l = 0.0
    for (b, h) in heads:
        rows = None if rows_per_head is None else sample_rows(case.N, rows_per_head, 17 * b + h)
        o_ref, l_ref = case.oracle_fwd(b, h, rows)
        sel = np.arange(case.N) if rows is None else rows
        worst_o = max(worst_o, float(np.abs(O_gpu[b, h][sel] - o_ref).max()))
        worst_l = max(worst_l, float(np.abs(L_gpu[b, h][sel] - l_ref).max()))
    print(f"[{label}] max|O-O_ref| = {worst_o:.3e}  max|LSE-LSE_ref| = {worst_l:.3e}")
    assert worst_o <= TOL_O, f"{label}: O error {worst_o}"
    assert worst_l <= TOL_LSE, f"{label}: LSE error {worst_l}"
    return worst_o, worst_l


def check_bwd(case, grads, heads, nq, nk, label, extra_k=None):
    """Relative L2 of dQ / dK / dV against the oracle on sampled rows of `heads` (all rows when
    nq / nk is None); `extra_k` adds key rows to every head's sample (e.g. whole key tiles)."""
    dQ, dK, dV = (bf16_to_f64(g) for g in grads)
    worst = {"dQ": 0.0, "dK": 0.0, "dV": 0.0}
    for (b, h) in heads:
        qr = None if nq is None else sample_rows(case.N, nq, 31 * b + h)
        kr = None if nk is None else sample_rows(case.N, nk, 37 * b + h + 1)
        if kr is not None and extra_k is not None:
            kr = np.unique(np.concatenate([kr, np.asarray(extra_k, dtype=np.int64)]))
        dq, dk, dv, _, _ = case.oracle_bwd(b, h, qr, kr)
        qs = np.arange(case.N) if qr is None else qr
        ks = np.arange(case.N) if kr is None else kr
        worst["dQ"] = max(worst["dQ"], rel_l2(dQ[b, h][qs], dq))
        worst["dK"] = max(worst["dK"], rel_l2(dK[b, h][ks], dk))
        worst["dV"] = max(worst["dV"], rel_l2(dV[b, h][ks], dv))
    print(f"[{label}] rel L2: " + "  ".join(f"{k} {v:.3e}" for k, v in worst.items()))
    for k, v in worst.items():
        assert v <= TOL_GRAD, f"{label}: {k} relative L2 error {v}"
    return worst


def all_heads(case):
    return [(b, h) for b in range(case.B) for h in range(case.H)]


# ---------------------------------------------------------------- workloads
def test_tiny_forward_and_backward_full():
    c = Case(1, 1, 128, 64, False, seed_workload=1, bwd=True)
    o, lse = c.fwd_gpu()
    check_fwd(c, o, lse, [(0, 0)], None, "tiny fwd")
    check_bwd(c, c.bwd_gpu(o, lse), [(0, 0)], None, None, "tiny bwd")


def test_forward_causal_2048():
    c = Case(4, 16, 2048, 128, True, seed_workload=2)
    o, lse = c.fwd_gpu()
    check_fwd(c, o, lse, all_heads(c), 160, "fwd causal B4 H16 N2048")


def test_forward_rescale_stress_8192():
    c = Case(2, 16, 8192, 128, False, seed_workload=3, stress=True)
    o, lse = c.fwd_gpu()
    check_fwd(c, o, lse, all_heads(c), 96, "fwd stress B2 H16 N8192")


def test_long_context_forward_backward_32768():
    c = Case(1, 16, 32768, 128, True, seed_workload=4, bwd=True)
    o, lse = c.fwd_gpu()
    check_fwd(c, o, lse, all_heads(c), 48, "fwd causal B1 H16 N32768")
    grads = c.bwd_gpu(o, lse)
    # heads 0, 7 and 15 run in different waves of the heaviest-first CTA order; the first and the
    # last key tile (rows 0..127 and N-128..N-1) are checked in full on each
    edge_keys = np.concatenate([np.arange(128), np.arange(c.N - 128, c.N)])
    check_bwd(c, grads, [(0, 0), (0, 7), (0, 15)], 64, 64, "bwd causal B1 H16 N32768", extra_k=edge_keys)
    # invariants over every head: sum_j dV_j = sum_i dO_i, sum_j dK_j = 0
    dK = bf16_to_f64(grads[1])
    dV = bf16_to_f64(grads[2])
    from exact_attention_159_b200 import inputs as I
    dO = I.bf16_bits_to_f64(c.bits["do"])
    for h in range(c.H):
        s_dv, s_do = dV[0, h].sum(0), dO[0, h].sum(0)
        assert rel_l2(s_dv, s_do) <= TOL_GRAD, f"head {h}: sum dV != sum dO"
        spread = np.sqrt((np.linalg.norm(dK[0, h], axis=1) ** 2).sum())
        assert np.linalg.norm(dK[0, h].sum(0)) <= 0.05 * spread, f"head {h}: sum dK != 0"


def test_causal_cta_groups_head_count_not_a_power_of_two():
    """30 heads of 4096 causal rows: the causal CTA order takes the heads in groups sized to the
    work per head and lowered to a divisor of the head count (15 heads per forward group, 6 per
    backward group here).  Every head and every query and key tile must still be computed once:
    each checked head has rows sampled in all of its query tiles and its first and last key tile
    checked in full."""
    c = Case(2, 15, 4096, 64, True, seed_workload=16, bwd=True)
    o, lse = c.fwd_gpu()
    heads = [(b, h) for b in range(2) for h in (0, 7, 14)]
    check_fwd(c, o, lse, heads, 64, "fwd causal B2 H15 N4096 d64")
    edge_keys = np.concatenate([np.arange(128), np.arange(c.N - 128, c.N)])
    check_bwd(c, c.bwd_gpu(o, lse), heads, 64, 64, "bwd causal B2 H15 N4096 d64", extra_k=edge_keys)


def test_causal_cta_groups_prime_head_count():
    """11 heads of 8192 causal rows: no divisor of 11 lies near the group size the work per head
    asks for (8 in the forward, 4 in the backward), so all 11 heads form one group."""
    c = Case(1, 11, 8192, 64, True, seed_workload=17, bwd=True)
    o, lse = c.fwd_gpu()
    heads = [(0, 0), (0, 5), (0, 10)]
    check_fwd(c, o, lse, heads, 64, "fwd causal B1 H11 N8192 d64")
    edge_keys = np.concatenate([np.arange(128), np.arange(c.N - 128, c.N)])
    check_bwd(c, c.bwd_gpu(o, lse), heads, 48, 48, "bwd causal B1 H11 N8192 d64", extra_k=edge_keys)


SWEEP = [(B, N, d, causal) for (B, N) in ((8, 2048), (2, 8192), (1, 16384)) for d in (64, 128)
         for causal in (False, True)]


@pytest.mark.parametrize("B,N,d,causal", SWEEP, ids=[f"B{b}-N{n}-d{d}-{'c' if c else 'f'}" for b, n, d, c in SWEEP])
def test_backward_sweep(B, N, d, causal):
    c = Case(B, 16, N, d, causal, seed_workload=5, bwd=True)
    o, lse = c.fwd_gpu()
    heads = [(0, 0), (B - 1, 7)]
    check_fwd(c, o, lse, heads, 48, f"sweep fwd B{B} N{N} d{d} causal={causal}")
    check_bwd(c, c.bwd_gpu(o, lse), heads, 48, 48, f"sweep bwd B{B} N{N} d{d} causal={causal}",
              extra_k=np.arange(N - 128, N))


# --------------------------------------------------------------- edge cases
EDGE = [(N, d, causal) for N in (1, 17, 127, 129, 200, 383) for d in (64, 128) for causal in (False, True)]


@pytest.mark.parametrize("N,d,causal", EDGE, ids=[f"N{n}-d{d}-{'c' if c else 'f'}" for n, d, c in EDGE])
def test_ragged_lengths_full(N, d, causal):
    c = Case(1, 2, N, d, causal, seed_workload=11, bwd=True)
    o, lse = c.fwd_gpu()
    check_fwd(c, o, lse, all_heads(c), None, f"ragged N{N} d{d} c{int(causal)}")
    check_bwd(c, c.bwd_gpu(o, lse), all_heads(c), None, None, f"ragged bwd N{N} d{d} c{int(causal)}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_several_tiles_and_heads_full(d, causal):
    c = Case(2, 3, 640, d, causal, seed_workload=12, bwd=True)
    o, lse = c.fwd_gpu()
    check_fwd(c, o, lse, all_heads(c), None, f"multi d{d} c{int(causal)}")
    check_bwd(c, c.bwd_gpu(o, lse), all_heads(c), None, None, f"multi bwd d{d} c{int(causal)}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("tau,poly", [(8.0, 4), (8.0, 2), (8.0, 1), (0.0, 0), (0.0, 4), (8.0, 0)])
def test_rescale_and_exp_variants_agree(tau, poly, d):
    c = Case(1, 4, 2048, d, False, seed_workload=3, stress=True)
    api.fa_set_softmax_options(8.0, -1)
    o_ref_gpu, lse_ref_gpu = c.fwd_gpu()
    try:
        api.fa_set_softmax_options(tau, poly)
        o, lse = c.fwd_gpu()
    finally:
        api.fa_set_softmax_options(8.0, -1)
    check_fwd(c, o, lse, all_heads(c), 128, f"variant tau={tau} poly={poly}")
    assert float((o.float() - o_ref_gpu.float()).abs().max()) <= TOL_O
    assert float((lse - lse_ref_gpu).abs().max()) <= TOL_LSE


def test_repeat_calls_deterministic():
    c = Case(1, 4, 1024, 128, True, seed_workload=13, bwd=True)
    o1, l1 = c.fwd_gpu()
    o2, l2 = c.fwd_gpu()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    g1 = c.bwd_gpu(o1, l1)
    g2 = c.bwd_gpu(o1, l1)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2])
    # dQ accumulates with fp32 atomics in varying order: equal up to one bf16 ulp
    assert float((g1[0].float() - g2[0].float()).abs().max()) <= 2.0 ** -6 * float(g1[0].float().abs().max())


def test_empty_problem_is_noop():
    lib = _lib.lib()
    q = torch.zeros(16, dtype=torch.bfloat16, device="cuda")
    o = torch.full((16,), 7.0, dtype=torch.bfloat16, device="cuda")
    l = torch.zeros(16, dtype=torch.float32, device="cuda")
    import ctypes
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    assert lib.fa_fwd(P(q), P(q), P(q), P(o), P(l), 0, 4, 128, 64, 0.125, 0, None) == 0
    torch.cuda.synchronize()
    assert float(o.float().min()) == 7.0


def test_unsupported_head_dim_launches_nothing():
    q = torch.zeros((1, 1, 128, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(_lib.FAError) as e:
        api.fa_fwd(q, q.clone(), q.clone())
    assert e.value.code == _lib.FA_ERR_UNSUPPORTED


# ------------------------------------------------ forward kernel variants
VARIANT_SHAPES = [(1, 2, 200, True), (2, 3, 640, False), (1, 2, 640, True), (1, 4, 1000, True), (1, 2, 1536, False),
                  (2, 2, 2048, True)]


@pytest.mark.parametrize("variant", [0, 1], ids=["single-cta", "cluster-pair"])
@pytest.mark.parametrize("B,H,N,causal", VARIANT_SHAPES, ids=[f"B{b}H{h}N{n}{'c' if c else 'f'}" for b, h, n, c in VARIANT_SHAPES])
def test_forward_variants_full(variant, B, H, N, causal):
    c = Case(B, H, N, 128, causal, seed_workload=14)
    api.fa_set_forward_variant(variant)
    try:
        o, lse = c.fwd_gpu()
    finally:
        api.fa_set_forward_variant(0)
    check_fwd(c, o, lse, all_heads(c), None if N <= 1000 else 160, f"variant {variant} B{B} H{H} N{N} c{int(causal)}")


def test_forward_variants_agree_at_full_size():
    c = Case(1, 16, 32768, 128, True, seed_workload=4)
    o0, l0 = c.fwd_gpu()
    api.fa_set_forward_variant(1)
    try:
        o1, l1 = c.fwd_gpu()
    finally:
        api.fa_set_forward_variant(0)
    assert float((o0.float() - o1.float()).abs().max()) <= 1e-2
    assert float((l0 - l1).abs().max()) <= 1e-3


# ----------------------------------------------- backward kernel variants
# (B, H, N, causal): one key tile (the pair's second tile lies past the end), odd and even tile
# counts, ragged tails, and several heads and batches
BWD_VARIANT_SHAPES = [(1, 1, 17, True), (1, 1, 128, True), (1, 2, 200, False), (1, 2, 256, True),
                      (2, 3, 640, False), (1, 2, 640, True), (1, 4, 1000, True), (1, 2, 1536, False),
                      (2, 2, 2048, True)]


@pytest.mark.parametrize("variant", [0, 1], ids=["single-cta", "cluster-pair"])
@pytest.mark.parametrize("B,H,N,causal", BWD_VARIANT_SHAPES,
                         ids=[f"B{b}H{h}N{n}{'c' if c else 'f'}" for b, h, n, c in BWD_VARIANT_SHAPES])
def test_backward_variants_full(variant, B, H, N, causal):
    c = Case(B, H, N, 128, causal, seed_workload=15, bwd=True)
    o, lse = c.fwd_gpu()
    api.fa_set_backward_variant(variant)
    try:
        grads = c.bwd_gpu(o, lse)
    finally:
        api.fa_set_backward_variant(0)
    full = N <= 1000
    check_bwd(c, grads, all_heads(c), None if full else 96, None if full else 96,
              f"bwd variant {variant} B{B} H{H} N{N} c{int(causal)}")


def test_backward_variants_agree_at_full_size():
    c = Case(1, 16, 32768, 128, True, seed_workload=4, bwd=True)
    o, lse = c.fwd_gpu()
    g0 = c.bwd_gpu(o, lse)
    api.fa_set_backward_variant(1)
    try:
        g1 = c.bwd_gpu(o, lse)
    finally:
        api.fa_set_backward_variant(0)
    check_bwd(c, g1, [(0, 0), (0, 11)], 64, 64, "bwd cluster-pair causal B1 H16 N32768")
    for a, b in zip(g0, g1):
        assert rel_l2(b.double().cpu().numpy(), a.double().cpu().numpy()) <= TOL_GRAD

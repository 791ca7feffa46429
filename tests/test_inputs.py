"""Seeded input generator: determinism, distribution, bf16 rounding (CPU)."""
import numpy as np
import torch

from exact_attention_159_b200 import inputs as I


def test_uniform_counter_slices_agree():
    a = I.uniform(1234, 0, 1000)
    b = I.uniform(1234, 500, 500)
    assert np.array_equal(a[500:], b)
    assert a.min() >= 0.0 and a.max() < 1.0
    assert not np.array_equal(a, I.uniform(1235, 0, 1000))


def test_normal_moments():
    z = I.normal(7, 400_000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1.0) < 0.01
    assert abs(np.mean(z ** 4) - 3.0) < 0.05   # Gaussian kurtosis


def test_bf16_rounding_matches_torch():
    r = np.random.default_rng(0)
    x = np.concatenate([r.standard_normal(100_000) * 10.0 ** r.integers(-8, 8, 100_000),
                        [0.0, -0.0, 1.0, 1.00390625, 1.005859375, 65504.0]])
    ours = I.f64_to_bf16_bits(x)
    ref = torch.tensor(x.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = I.bf16_bits_to_f64(ours)
    assert np.array_equal(back, torch.tensor(x.astype(np.float32)).to(torch.bfloat16).double().numpy())


def test_attention_inputs_shapes_and_stress():
    t = I.attention_inputs(3, 1, 2, 256, 64, stress=True, with_do=True)
    for k in ("q", "k", "v", "do"):
        assert t[k].shape == (1, 2, 256, 64) and t[k].dtype == np.uint16
    q = I.bf16_bits_to_f64(t["q"]).reshape(-1, 64)
    plain = I.bf16_bits_to_f64(I.attention_inputs(3, 1, 2, 256, 64)["v"])
    assert np.array_equal(plain, I.bf16_bits_to_f64(t["v"]))
    # the stress offsets along u are visible as a large common component
    u = I.normal(I.seed_for(3, "u"), 64); u /= np.linalg.norm(u)
    proj = q @ u
    assert 2.5 < proj.mean() < 5.5 and proj.max() > 6.0


def test_head_inputs_equal_slices_of_the_full_tensors():
    B, H, N, d = 2, 3, 96, 64
    for stress in (False, True):
        full = I.attention_inputs(7, B, H, N, d, stress=stress, with_do=True)
        for (b, h) in ((0, 0), (1, 2), (0, 2)):
            one = I.head_inputs(7, B, H, N, d, b, h, stress=stress, with_do=True)
            for k in ("q", "k", "v", "do"):
                assert np.array_equal(one[k], full[k][b, h]), (stress, b, h, k)

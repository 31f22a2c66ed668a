"""Input generator: determinism, shapes, bf16 rounding, feature layout."""
import numpy as np
import torch

import synthetic as syn


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.005859375, 3.0e-39, -65504.0], np.float32)])
    ours = syn.f32_to_bf16_bits_reference(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    assert np.array_equal(syn.f32_to_bf16_bits(x), ours)          # the fast path gives the same bits
    back = syn.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_tiny_inputs_deterministic():
    a = syn.make_inputs(1)
    b = syn.make_inputs(1)
    assert a["q"].shape == (1, 1024, 2, 64) and a["q"].dtype == np.float32
    for n in "qkv":
        assert np.array_equal(a[n], b[n])
    assert list(a["s"]) == [0.5, 3.0]
    c = syn.make_inputs(1, sub=1)
    assert not np.array_equal(a["q"], c["q"])


def test_feature_layout():
    f = syn.features(3, 4, 5, 128).reshape(3, 4, 5, 128)
    # t group: pair 0 is (sin t, cos t); y group starts at dim 44; x group at 86
    assert np.allclose(f[2, 0, 0, 0], np.sin(2.0)) and np.allclose(f[2, 0, 0, 1], np.cos(2.0))
    assert np.allclose(f[0, 3, 0, 44], np.sin(3.0)) and np.allclose(f[0, 0, 4, 87], np.cos(4.0))
    assert np.allclose(f[..., 0::2] ** 2 + f[..., 1::2] ** 2, 1.0, atol=1e-6)


def test_small_bf16_variant():
    w = syn.workload(2, T=2, Hs=6, Ws=10, H=3)
    x = syn.make_inputs(w)
    assert x["q"].dtype == np.uint16 and x["q"].shape == (1, 120, 3, 128)
    assert np.all((x["c"] >= 0) & (x["c"] <= 2)) and np.all((x["s"] >= 0.25) & (x["s"] <= 4))

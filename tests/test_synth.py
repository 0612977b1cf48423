"""Host-side checks of the seeded input generator (no GPU)."""
import numpy as np
import torch

from tensor_transformer_layer_linear_b200 import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 3,
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0], np.float32)])
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = synth.bf16_bits_to_f64(ours)
    assert np.array_equal(back, torch.from_numpy(ours.view(np.int16)).view(torch.bfloat16)
                          .to(torch.float64).numpy())


def test_inputs_are_seeded_and_shaped():
    cfg = synth.config("mlp_32x1024_f4096_n2")
    a, b = synth.make_inputs(cfg, 0), synth.make_inputs(cfg, 0)
    assert all(np.array_equal(a[k], b[k]) for k in a)
    assert a["X"].shape == (32, 1024) and a["A"].shape == (1024, 4096)
    assert a["B"].shape == (4096, 1024) and not a["b1"].any()
    c = synth.make_inputs(cfg, 1)
    assert not np.array_equal(a["X"], c["X"])
    x = synth.bf16_bits_to_f64(a["X"])
    assert abs(x.std() - 1.0) < 0.02


def test_sample_rows():
    rows = synth.sample_rows(2, 2048)
    assert rows[0] == 0 and rows[-1] == 4095 and 2047 in rows and 2048 in rows
    assert len(rows) == 2 * (2048 // 64) + 2

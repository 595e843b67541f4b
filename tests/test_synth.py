"""Checks on the seeded input generators (no method arithmetic lives there)."""

import numpy as np
import torch

import synth


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100_000).astype(np.float32) * 0.02,
                        np.array([0.0, -0.0, 1.0, 3.0e38, -1e-40, 1.00390625, 1.01171875],
                                 dtype=np.float32)])
    bits, vals = synth.bf16_round(a)
    ref = torch.from_numpy(a).to(torch.bfloat16)
    np.testing.assert_array_equal(bits, ref.view(torch.int16).numpy().view(np.uint16))
    np.testing.assert_array_equal(vals, ref.float().numpy())
    np.testing.assert_array_equal(synth.bf16_bits_to_f32(bits), vals)


def test_k_counts_match_the_workloads():
    assert synth.ffn_k(1376, 70) == 413
    assert [synth.ffn_k(14336, s) for s in (0, 50, 60, 70)] == [14336, 7168, 5734, 4301]
    assert synth.ffn_k(17408, 70) == 5222
    assert synth.ffn_k(28672, 70) == 8602
    assert [synth.get_config(n).n_outliers for n in
            ("tiny", "llama3_8b", "qwen3_14b", "llama3_70b")] == [5, 20, 26, 41]


def test_layers_are_seeded_and_reproducible():
    a = synth.make_layer("tiny", n_tokens=3)
    b = synth.make_layer("tiny", n_tokens=3)
    np.testing.assert_array_equal(a.w_gate_bits, b.w_gate_bits)
    np.testing.assert_array_equal(a.x_eval, b.x_eval)
    assert a.w_gate.shape == (512, 1376) and a.w_down.shape == (1376, 512)
    assert a.x_cal.shape == (256, 512) and a.x_eval.dtype == np.float32
    # outlier channels carry the configured scale in every token
    other = np.setdiff1d(np.arange(512), a.outliers)
    assert np.abs(a.x_cal[:, a.outliers]).mean() > 10 * np.abs(a.x_cal[:, other]).mean()
    c = synth.make_layer("tiny", layer=1, draw_tokens=False)
    assert not np.array_equal(a.w_gate_bits, c.w_gate_bits) and c.x_eval is None

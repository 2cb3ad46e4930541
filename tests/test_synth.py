"""The seeded input generator: bf16 rounding, shapes, draw order, counted work."""
import numpy as np
import torch

from vision_transformer_encoder_dsv4v_b200 import synth


def test_bf16_rounding_matches_torch():
    a = np.random.default_rng(0).standard_normal(100000, dtype=np.float32) * 3
    a[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 65504.0]   # ties to even
    bits = synth.bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    np.testing.assert_array_equal(synth.bf16_to_f32(bits), torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_workload_shapes_and_flops():
    w2, w3, w4 = synth.workload(2), synth.workload(3), synth.workload(4)
    assert w2.n_patches == 784 and w3.n_patches == 3562 and w4.n_tokens == 196
    assert abs(synth.algorithmic_flops(w2) / 1e9 - 22.66) < 0.01
    assert abs(synth.algorithmic_flops(w3) / 1e9 - 104.69) < 0.01
    assert abs(synth.algorithmic_flops(w4) / 1e9 - 731.65) < 0.01
    w5 = synth.workload(5)
    assert len(w5.grids) == 16 and (64, 64) in w5.grids and 20000 <= w5.n_patches <= 30000
    assert all(8 <= a <= 64 and 8 <= b <= 64 for a, b in w5.grids)


def test_draw_order_prefix_property():
    wl = synth.workload(1)
    full = synth.draw(wl)
    assert full.x.values.shape == (24, 64) and full.x.bits is None
    assert full.w_align.values.shape == (128, 256) and full.final_norm_w is None
    wl4 = synth.workload(4)
    two = synth.draw(wl4, n_layers=2)
    one = synth.draw(wl4, n_layers=1)
    np.testing.assert_array_equal(two.layers[0]["w_down"].bits, one.layers[0]["w_down"].bits)
    np.testing.assert_array_equal(two.x.bits, one.x.bits)
    assert two.w_align is None

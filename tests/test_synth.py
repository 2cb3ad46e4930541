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


def _layouts():
    # stand-in layouts of distinct lengths (the generator only places them)
    return [np.array([1] + [0] * (k + 1) + [2], dtype=np.int32) for k in range(7)]


def test_place_spans_keeps_every_layout_intact_and_in_order():
    lays = _layouts()
    for balance in (False, True):
        t = synth.place_spans(lays, 3, 40, seed=5, max_gap=3, balance=balance)
        found = []
        for row in t:
            starts = np.flatnonzero(row == 1)
            ends = np.flatnonzero(row == 2)
            for a, e in zip(starts, ends):
                found.append(row[a:e + 1])
        assert len(found) == len(lays)
        for f, lay in zip(found, lays):
            np.testing.assert_array_equal(f, lay)
        assert set(np.unique(t)) <= {-1, 0, 1, 2}
    # balance: image i sits in sequence floor(i * n_seqs / n_images)
    t = synth.place_spans(lays, 3, 40, seed=5, max_gap=3, balance=True)
    assert [int((row == 1).sum()) for row in t] == [3, 2, 2]


def test_place_spans_pad_every_and_errors():
    lays = _layouts()
    t = synth.place_spans(lays, 2, 60, seed=1, max_gap=0, pad_every=3)
    assert int((t == 4).sum()) == 2  # images 2 and 5
    for row in t:  # each filler sits right before an image_end
        for p in np.flatnonzero(row == 4):
            assert row[p + 1] == 2
    try:
        synth.place_spans(lays, 1, 10, seed=1)
    except ValueError:
        pass
    else:
        raise AssertionError("an overfull placement must raise")


def test_bench_bridge_stream_is_a_valid_layout():
    # the stream the benchmark's bridge extra builds (the library's host N-layout of the
    # high-resolution batch, 4 x 8192 positions) is accepted by the oracle's merge and span rules
    from oracle import dsv4v_oracle as O
    from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
    grids = synth.workload(5).grids
    types = synth.place_spans([A.dsv4v_image_layout(h, w, 2) for h, w in grids], 4, 8192, seed=21, pad_every=4,
                              balance=True)
    per = [-(-h // 2) * -(-w // 2) for h, w in grids]
    e = 2
    out = O.merge_image_embeddings(np.zeros(types.shape + (e,)), types, np.ones((sum(per), e)),
                                   np.full((4, e), 2.0), per)
    assert int((out[..., 0] == 1.0).sum()) == sum(per)
    assert [len(O.image_spans(row)) for row in types] == [4, 4, 4, 4]

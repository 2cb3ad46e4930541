"""Pins of the fp64 oracle to facts other than itself: closed forms, invariants, brute force on
tiny inputs and hand-written tables.  CPU only.

Each test names the mistake it would catch in the oracle (a dropped term, a wrong sign, index or
scale, a transposed operand)."""
import cmath
import itertools
import math
import os

import numpy as np
import pytest

from oracle import dsv4v_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


# ------------------------------------------------------------------------------- RMSNorm
def test_rmsnorm_constant_row_closed_form():
    # y = w c / sqrt(c^2 + eps) for a constant row; catches sum-vs-mean and a misplaced eps.
    d, c, eps = 37, -1.7, 1e-6
    w = RNG.normal(size=d)
    y = O.rmsnorm(np.full((1, d), c), w, eps)
    np.testing.assert_allclose(y[0], w * c / math.sqrt(c * c + eps), rtol=1e-14)


def test_rmsnorm_unit_weight_rms():
    # with w = 1: rms(y) = sqrt(ms / (ms + eps)).
    x = RNG.normal(size=(5, 64)) * 0.01
    eps = 1e-4
    y = O.rmsnorm(x, np.ones(64), eps)
    ms = np.mean(x * x, axis=1)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, axis=1)), np.sqrt(ms / (ms + eps)), rtol=1e-13)


def test_rmsnorm_scale_invariance_and_direct_weight():
    # eps = 0: y(a x) = sign(a) y(x); w = 0 gives 0 (catches a "1 + w" scale).
    x = RNG.normal(size=(3, 16))
    w = RNG.normal(size=16)
    np.testing.assert_allclose(O.rmsnorm(7.5 * x, w, 0.0), O.rmsnorm(x, w, 0.0), rtol=1e-13)
    np.testing.assert_allclose(O.rmsnorm(-2.0 * x, w, 0.0), -O.rmsnorm(x, w, 0.0), rtol=1e-13)
    assert np.all(O.rmsnorm(x, np.zeros(16), 1e-6) == 0.0)


def test_rmsnorm_hand_value():
    # x = (3, 4): mean square 12.5; eps = 0; w = (1, 2) -> (3, 8) / sqrt(12.5).
    y = O.rmsnorm(np.array([[3.0, 4.0]]), np.array([1.0, 2.0]), 0.0)
    np.testing.assert_allclose(y[0], [0.848528137423857, 2.262741699796952], rtol=1e-14)


# ------------------------------------------------------------------------------- RoPE table
def test_rope_origin_is_identity_and_axes_separate():
    cos, sin = O.vision_cos_sin(5, 7, 16, 10000.0)
    assert np.all(cos[0] == 1.0) and np.all(sin[0] == 0.0)          # patch (0, 0)
    c1, s1 = O.vision_cos_sin(1, 9, 16, 10000.0)                    # one row: row half identity
    assert np.all(c1[:, :8] == 1.0) and np.all(s1[:, :8] == 0.0)
    c2, s2 = O.vision_cos_sin(9, 1, 16, 10000.0)                    # one column: column half identity
    assert np.all(c2[:, 8:] == 1.0) and np.all(s2[:, 8:] == 0.0)
    # row half depends on h only, column half on w only (patch p = h*n_w + w)
    for p, q in itertools.combinations(range(35), 2):
        hp, wp, hq, wq = p // 7, p % 7, q // 7, q % 7
        if hp == hq:
            np.testing.assert_array_equal(cos[p, :8], cos[q, :8])
        if wp == wq:
            np.testing.assert_array_equal(cos[p, 8:], cos[q, 8:])


def test_rope_frequency_schedule():
    # unit step in h: angle of pair k is theta^(-k/(dim/2)); the first pair turns by 1 rad, the
    # ratio between neighbours is theta^(-1/(dim/2)) (catches a theta^(-2k/dim) schedule).
    dim, theta = 32, 10000.0
    cos, sin = O.vision_cos_sin(2, 1, dim, theta)
    ang = np.arctan2(sin[1, :16], cos[1, :16])
    assert abs(ang[0] - 1.0) < 1e-15
    np.testing.assert_allclose(ang[1:] / ang[:-1], theta ** (-1.0 / 16), rtol=1e-12)
    # angles are linear in the position: angle(h=3) = 3 angle(h=1) (mod 2 pi)
    c3, s3 = O.vision_cos_sin(4, 1, dim, theta)
    z1 = c3[1, :16] + 1j * s3[1, :16]
    z3 = c3[3, :16] + 1j * s3[3, :16]
    np.testing.assert_allclose(z1 ** 3, z3, atol=1e-13)


def test_rotary_matches_complex_multiplication():
    # brute force through another formulation: pair (x_j, x_{j+hd/2}) as x_j + i x_{j+hd/2},
    # multiplied by exp(i angle_j).  Catches a sign error or an interleaved-pair convention.
    n_h, n_w, hd = 3, 4, 8
    cos, sin = O.vision_cos_sin(n_h, n_w, hd // 2, 100.0)
    x = RNG.normal(size=(n_h * n_w, 2, hd))
    y = O.apply_vision_rotary(x, cos, sin)
    for p in range(n_h * n_w):
        for h in range(2):
            for j in range(hd // 2):
                ang = math.atan2(sin[p, j], cos[p, j])
                z = complex(x[p, h, j], x[p, h, j + hd // 2]) * cmath.exp(1j * ang)
                assert abs(y[p, h, j] - z.real) < 1e-13
                assert abs(y[p, h, j + hd // 2] - z.imag) < 1e-13


def test_rotary_preserves_pair_norms():
    cos, sin = O.vision_cos_sin(6, 5, 8, 10000.0)
    x = RNG.normal(size=(30, 3, 16))
    y = O.apply_vision_rotary(x, cos, sin)
    nx = x[..., :8] ** 2 + x[..., 8:] ** 2
    ny = y[..., :8] ** 2 + y[..., 8:] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-14)


def test_rotary_relative_position_property():
    # <R(p) q, R(p') k> depends only on (h - h', w - w'): shift both patches by (dh, dw).
    n, hd = 16, 16
    cos, sin = O.vision_cos_sin(n, n, hd // 2, 10000.0)
    q = RNG.normal(size=(1, 1, hd))
    k = RNG.normal(size=(1, 1, hd))

    def dot(p, pp):
        rq = O.apply_vision_rotary(q, cos[p:p + 1], sin[p:p + 1])
        rk = O.apply_vision_rotary(k, cos[pp:pp + 1], sin[pp:pp + 1])
        return float(np.sum(rq * rk))

    for (h, w, h2, w2, dh, dw) in [(1, 2, 5, 9, 3, 4), (10, 0, 2, 3, 5, 12), (0, 0, 15, 15, -0, -0),
                                   (7, 7, 7, 7, 8, -7), (3, 11, 12, 1, 2, 3)]:
        a = dot(h * n + w, h2 * n + w2)
        b = dot((h + dh) * n + (w + dw), (h2 + dh) * n + (w2 + dw))
        assert abs(a - b) < 1e-12 * max(1.0, abs(a))
    # and the rotation is not trivial: a different offset gives a different product
    assert abs(dot(0, 1) - dot(0, 2)) > 1e-6


# ------------------------------------------------------------------------------- fused projection + rotation
def _qkv_rope_checks(qkv_rope):
    """Facts about the projection-plus-rotation of one 6x6 image that hold for the stated
    definition [vision-API, DeepseekV4VisionAttention, apply_vision_rotary]; returns the names of
    the ones that fail.  (a) with one y row shared by every patch, q_p . k_p' of each head depends
    only on (h - h', w - w'): fails when q or k is left unrotated; (b) with that shared row every
    v row is equal: fails when v is rotated; (c) with distinct random y, q and k equal the
    rotation, written out by hand below, of y . W[0:D]^T and y . W[D:2D]^T and v equals
    y . W[2D:3D]^T: fails on a swap or reorder of the q | k | v blocks."""
    n, d, nh = 6, 16, 2
    hd = d // nh
    rng = np.random.default_rng(77)
    cos, sin = O.vision_cos_sin(n, n, hd // 2, 100.0)
    w = rng.normal(size=(3 * d, d))
    failed = []
    y_same = np.tile(rng.normal(size=(1, d)), (n * n, 1))
    q, k, v = qkv_rope(y_same, w, cos, sin, nh)

    def dot(h, p, pp):
        return float(np.dot(q[p, h], k[pp, h]))

    rel_ok = True
    for h in range(nh):
        for (a, b, a2, b2, dh, dw) in [(0, 1, 3, 4, 2, 1), (5, 0, 3, 2, -3, 3), (2, 4, 0, 5, 1, -4),
                                       (1, 3, 4, 0, 1, 2)]:
            assert all(0 <= t < n for t in (a + dh, a2 + dh, b + dw, b2 + dw))
            x0 = dot(h, a * n + b, a2 * n + b2)
            x1 = dot(h, (a + dh) * n + (b + dw), (a2 + dh) * n + (b2 + dw))
            rel_ok &= abs(x0 - x1) < 1e-10 * max(1.0, abs(x0))
    if not rel_ok:
        failed.append("relative position")
    if not np.allclose(v, v[:1], rtol=0, atol=1e-12):
        failed.append("v rows equal")
    y = rng.normal(size=(n * n, d))
    q, k, v = qkv_rope(y, w, cos, sin, nh)
    blocks_ok = True
    for p in range(n * n):
        for h in range(nh):
            for which, got in ((0, q), (1, k)):
                lin = [sum(y[p, c] * w[which * d + h * hd + j, c] for c in range(d)) for j in range(hd)]
                for j in range(hd // 2):
                    c_, s_ = cos[p, j], sin[p, j]
                    want_lo = lin[j] * c_ - lin[j + hd // 2] * s_
                    want_hi = lin[j + hd // 2] * c_ + lin[j] * s_
                    blocks_ok &= abs(got[p, h, j] - want_lo) < 1e-11 and abs(got[p, h, j + hd // 2] - want_hi) < 1e-11
            for j in range(hd):
                want_v = sum(y[p, c] * w[2 * d + h * hd + j, c] for c in range(d))
                blocks_ok &= abs(v[p, h, j] - want_v) < 1e-11
    if not blocks_ok:
        failed.append("q | k | v blocks")
    return failed


def test_qkv_rope_rotates_q_and_k_in_block_order():
    assert _qkv_rope_checks(O.qkv_rope) == []


def _planted(kind):
    """Copies of the oracle's projection with one plausible mistake each (planted here, on the
    CPU, to show that the checks above catch it)."""
    def f(y, wqkv, cos, sin, n_heads):
        y = np.asarray(y, dtype=np.float64)
        d = y.shape[1]
        hd = d // n_heads
        qkv = y @ np.asarray(wqkv, dtype=np.float64).T
        q = qkv[:, :d].reshape(-1, n_heads, hd)
        k = qkv[:, d:2 * d].reshape(-1, n_heads, hd)
        v = qkv[:, 2 * d:].reshape(-1, n_heads, hd)
        rot = lambda t: O.apply_vision_rotary(t, cos, sin)
        if kind == "rotate q only":
            return rot(q), k, v
        if kind == "rotate k only":
            return q, rot(k), v
        if kind == "swap q and k":
            return rot(k), rot(q), v
        if kind == "rotate v too":
            return rot(q), rot(k), rot(v)
        if kind == "k and v blocks swapped":
            return rot(q), rot(v), k
        raise ValueError(kind)
    return f


@pytest.mark.parametrize("kind,caught_by", [("rotate q only", "relative position"),
                                            ("rotate k only", "relative position"),
                                            ("swap q and k", "q | k | v blocks"),
                                            ("rotate v too", "v rows equal"),
                                            ("k and v blocks swapped", "q | k | v blocks")])
def test_qkv_rope_checks_catch_planted_mistakes(kind, caught_by):
    assert caught_by in _qkv_rope_checks(_planted(kind))


# ------------------------------------------------------------------------------- attention
def _naive_attention(q, k, v):
    """Pure-Python loops, exp without max subtraction, scale 1/sqrt(hd)."""
    n, nh, hd = q.shape
    out = np.zeros((n, nh * hd))
    for h in range(nh):
        for i in range(n):
            w = [math.exp(sum(q[i, h, c] * k[j, h, c] for c in range(hd)) / math.sqrt(hd)) for j in range(n)]
            z = sum(w)
            for c in range(hd):
                out[i, h * hd + c] = sum(w[j] * v[j, h, c] for j in range(n)) / z
    return out


def test_attention_brute_force():
    q, k, v = (RNG.normal(size=(7, 2, 4)) for _ in range(3))
    np.testing.assert_allclose(O.attention_one_image(q, k, v), _naive_attention(q, k, v), rtol=1e-12, atol=1e-14)


def test_attention_two_key_closed_form_pins_scale():
    # one query a e_0, keys 0 and s e_0: p_1 = 1 / (1 + exp(-a s / sqrt(hd))).
    hd, a, s = 16, 1.5, 2.0
    q = np.zeros((1, 1, hd)); q[0, 0, 0] = a
    k = np.zeros((2, 1, hd)); k[1, 0, 0] = s
    v = np.zeros((2, 1, hd)); v[1, 0, 3] = 1.0
    qq = np.concatenate([q, q])  # two queries, identical
    out = O.attention_one_image(qq, k, v)
    assert abs(out[0, 3] - 1.0 / (1.0 + math.exp(-a * s / 4.0))) < 1e-15


def test_attention_rows_sum_to_one_and_special_cases():
    q, k, v = (RNG.normal(size=(9, 3, 8)) for _ in range(3))
    for h in range(3):
        p = O.attention_probs(q[:, h], k[:, h])
        np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)
        assert np.all(p > 0)
    v_same = np.broadcast_to(v[:1], v.shape)
    np.testing.assert_allclose(O.attention_one_image(q, k, v_same), np.tile(v[0].reshape(1, -1), (9, 1)), rtol=1e-13)
    zero_q = np.zeros_like(q)
    np.testing.assert_allclose(O.attention_one_image(zero_q, k, v), np.tile(v.mean(axis=0).reshape(1, -1), (9, 1)), rtol=1e-12)


def test_attention_permutation_properties():
    q, k, v = (RNG.normal(size=(11, 2, 8)) for _ in range(3))
    out = O.attention_one_image(q, k, v)
    perm = RNG.permutation(11)
    np.testing.assert_allclose(O.attention_one_image(q, k[perm], v[perm]), out, rtol=1e-12)   # keys
    np.testing.assert_allclose(O.attention_one_image(q[perm], k, v), out[perm], rtol=1e-12)   # queries


def test_attention_packed_isolation():
    grids = [(2, 3), (1, 1), (3, 2)]
    q, k, v = (RNG.normal(size=(13, 2, 4)) for _ in range(3))
    out = O.attention_packed(q, k, v, grids)
    np.testing.assert_allclose(out[:6], O.attention_one_image(q[:6], k[:6], v[:6]), rtol=1e-14)
    np.testing.assert_allclose(out[6:7], v[6].reshape(1, -1), rtol=1e-14)   # a 1-patch image sees itself
    np.testing.assert_allclose(out[7:], O.attention_one_image(q[7:], k[7:], v[7:]), rtol=1e-14)


# ------------------------------------------------------------------------------- MLP
def test_silu_and_mlp_closed_forms():
    assert O.silu(0.0) == 0.0
    z = RNG.normal(size=20) * 4
    np.testing.assert_allclose(O.silu(z) - O.silu(-z), z, rtol=1e-13)          # z sigma(z) + z sigma(-z) = z
    # scalar SwiGLU: y = 2, gate 1.5, up -0.5, down 3 -> silu(3) * (-1) * 3, silu(3) = 3 / (1 + e^-3)
    out = O.mlp(np.array([[2.0]]), np.array([[1.5]]), np.array([[-0.5]]), np.array([[3.0]]))
    assert abs(out[0, 0] - (-3.0 * 3.0 / (1.0 + math.exp(-3.0)))) < 1e-14
    # the gate goes through silu, the up projection does not (catches swapped gate/up)
    out2 = O.mlp(np.array([[2.0]]), np.array([[-0.5]]), np.array([[1.5]]), np.array([[3.0]]))
    assert abs(out2[0, 0] - (3.0 * 3.0 * (-1.0) / (1.0 + math.exp(1.0)))) < 1e-14


# ------------------------------------------------------------------------------- block / tower
def _layer(d, f, rng, zero=()):
    lay = dict(norm1_w=1 + 0.1 * rng.normal(size=d), wqkv=0.2 * rng.normal(size=(3 * d, d)),
               wo=0.2 * rng.normal(size=(d, d)), norm2_w=1 + 0.1 * rng.normal(size=d),
               w_gate=0.2 * rng.normal(size=(f, d)), w_up=0.2 * rng.normal(size=(f, d)),
               w_down=0.2 * rng.normal(size=(d, f)))
    for z in zero:
        lay[z] = np.zeros_like(lay[z])
    return lay


GRIDS = [(3, 4), (2, 2)]


def test_block_zero_projections_is_identity():
    d, f, nh = 16, 24, 2
    x = RNG.normal(size=(16, d))
    cos, sin = O.packed_cos_sin(GRIDS, d // nh // 2, 10000.0)
    for zero in [("wqkv", "wo", "w_gate", "w_up", "w_down"), ("wo", "w_down")]:
        out = O.block_forward(x, _layer(d, f, RNG, zero), cos, sin, GRIDS, nh)
        np.testing.assert_array_equal(out, x)


def test_block_value_block_position_and_isolation():
    # q block = 0 -> every score 0 -> uniform attention over the image; v block = identity and
    # wo = identity -> attention branch = per-image mean of norm1(x).  Pins v as the third
    # block of wqkv and the per-image isolation; MLP off.
    d, f, nh = 8, 8, 2
    x = RNG.normal(size=(16, d))
    lay = _layer(d, f, RNG, ("w_gate", "w_up", "w_down"))
    lay["wqkv"][:d] = 0.0
    lay["wqkv"][2 * d:] = np.eye(d)
    lay["wo"] = np.eye(d)
    cos, sin = O.packed_cos_sin(GRIDS, d // nh // 2, 10000.0)
    out = O.block_forward(x, lay, cos, sin, GRIDS, nh)
    y = O.rmsnorm(x, lay["norm1_w"])
    want = x.copy()
    want[:12] += y[:12].mean(axis=0)
    want[12:] += y[12:].mean(axis=0)
    np.testing.assert_allclose(out, want, rtol=1e-13)
    # same with the k block zero instead of q (scores 0 again)
    lay["wqkv"][:d] = 0.3 * RNG.normal(size=(d, d))
    lay["wqkv"][d:2 * d] = 0.0
    np.testing.assert_allclose(O.block_forward(x, lay, cos, sin, GRIDS, nh), want, rtol=1e-13)


def test_block_mlp_only_branch():
    d, f, nh = 8, 12, 2
    x = RNG.normal(size=(16, d))
    lay = _layer(d, f, RNG, ("wqkv",))   # v = 0 -> attention branch 0
    cos, sin = O.packed_cos_sin(GRIDS, d // nh // 2, 10000.0)
    out = O.block_forward(x, lay, cos, sin, GRIDS, nh)
    y = O.rmsnorm(x, lay["norm2_w"])
    h = np.zeros((16, f))
    for p in range(16):   # explicit loops instead of matmuls
        for j in range(f):
            g = sum(y[p, c] * lay["w_gate"][j, c] for c in range(d))
            u = sum(y[p, c] * lay["w_up"][j, c] for c in range(d))
            h[p, j] = g / (1 + math.exp(-g)) * u
    want = x + np.array([[sum(h[p, j] * lay["w_down"][c, j] for j in range(f)) for c in range(d)] for p in range(16)])
    np.testing.assert_allclose(out, want, rtol=1e-12)


def test_tower_composition():
    d, f, nh = 16, 16, 2
    x = RNG.normal(size=(16, d))
    layers = [_layer(d, f, RNG) for _ in range(3)]
    fn = 1 + 0.1 * RNG.normal(size=d)
    cos, sin = O.packed_cos_sin(GRIDS, d // nh // 2, 10000.0)
    want = x
    for lay in layers:
        want = O.block_forward(want, lay, cos, sin, GRIDS, nh)
    np.testing.assert_allclose(O.tower_forward(x, layers, None, GRIDS, nh), want, rtol=1e-13)
    np.testing.assert_allclose(O.tower_forward(x, layers, fn, GRIDS, nh), O.rmsnorm(want, fn), rtol=1e-13)
    # layer order matters
    assert not np.allclose(O.tower_forward(x, layers[::-1], None, GRIDS, nh), want)


# ------------------------------------------------------------------------------- aligner
def _read_table(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            if line.strip() and not line.startswith("#"):
                rows.append([int(t) for t in line.split()])
    return rows


@pytest.mark.parametrize("grid,name", [((4, 6), "aligner_4x6_r2.txt"), ((3, 5), "aligner_3x5_r2.txt")])
def test_aligner_merge_hand_table(grid, name):
    n_h, n_w = grid
    p = n_h * n_w
    # two channels: (p+1, -(p+1)) so zero padding, patch 0 and the channel order are all visible
    x = np.stack([np.arange(1, p + 1), -np.arange(1, p + 1)], axis=1).astype(float)
    merged, cu_tok = O.aligner_merge(x, [grid], 2)
    table = _read_table(name)
    assert merged.shape == (len(table), 8) and list(cu_tok) == [0, len(table)]
    for t, row in enumerate(table):
        i, j, slots = row[0], row[1], row[2:]
        assert t == i * (-(-n_w // 2)) + j                       # tokens row-major
        for s, patch in enumerate(slots):
            want = [0.0, 0.0] if patch < 0 else [patch + 1.0, -(patch + 1.0)]
            assert list(merged[t, 2 * s:2 * s + 2]) == want, (t, s)


def test_aligner_projection_and_token_counts():
    d = 4
    grids = [(4, 6), (3, 5)]
    x = RNG.normal(size=(39, d))
    merged, cu_tok = O.aligner_merge(x, grids, 2)
    assert list(cu_tok) == [0, 6, 12]
    wa = np.zeros((4 * d, 4 * d))
    wa[np.arange(4 * d), np.arange(4 * d)] = 1.0                   # identity projection
    out, _ = O.aligner_forward(x, wa, grids, 2)
    np.testing.assert_array_equal(out, merged)
    # the validation grids of the pull request: token counts ceil(n_h/2) * ceil(n_w/2)
    for (n_h, n_w), t in [((28, 28), 196), ((27, 37), 266), ((37, 27), 266), ((10, 78), 195), ((112, 7), 224)]:
        _, cu = O.aligner_merge(np.zeros((n_h * n_w, 1)), [(n_h, n_w)], 2)
        assert cu[-1] == t


def test_cu_from_grids():
    assert list(O.cu_from_grids([(27, 37), (37, 27), (10, 78), (112, 7)])) == [0, 999, 1998, 2778, 3562]


def test_patch_embed_flatten_order_and_bias():
    """One-hot pixels pin the flatten order (channel, row, column); zero pixels give the bias;
    the map is linear."""
    rng = np.random.default_rng(5)
    ph, pw, d = 3, 4, 7
    w = rng.normal(size=(d, 3 * ph * pw))
    b = rng.normal(size=d)
    for c, i, j in [(0, 0, 0), (1, 2, 3), (2, 1, 0), (2, 2, 3)]:
        x = np.zeros((1, 3, ph, pw))
        x[0, c, i, j] = 1.0
        np.testing.assert_allclose(O.patch_embed(x, w)[0], w[:, c * ph * pw + i * pw + j], rtol=0, atol=0)
        np.testing.assert_allclose(O.patch_embed(x, w, b)[0], w[:, c * ph * pw + i * pw + j] + b, rtol=0, atol=1e-15)
    np.testing.assert_allclose(O.patch_embed(np.zeros((2, 3, ph, pw)), w, b), np.stack([b, b]), rtol=0, atol=0)
    x1, x2 = rng.normal(size=(5, 3, ph, pw)), rng.normal(size=(5, 3, ph, pw))
    np.testing.assert_allclose(O.patch_embed(2.0 * x1 - x2, w), 2.0 * O.patch_embed(x1, w) - O.patch_embed(x2, w),
                               rtol=1e-12, atol=1e-12)
    # one patch written out by hand: 3 x 1 x 1 pixels (r, g, b) = (1, 2, 3), w = rows [1 0 0], [1 1 1]
    np.testing.assert_allclose(O.patch_embed(np.array([[[[1.0]], [[2.0]], [[3.0]]]]),
                                             np.array([[1.0, 0.0, 0.0], [1.0, 1.0, 1.0]]), np.array([0.5, -1.0])),
                               [[1.5, 5.0]], rtol=0, atol=0)


def test_patch_merger_structure_matches_the_stated_parameter_count():
    """The pages give 40,119,040 parameters for the projector that merges 2x2 groups of 1152-wide
    patches (4608) into the 4096-wide token space: only LayerNorm(1152) + two biased Linears fits."""
    assert O.patch_merger_params(1152, 2, 4096) == 40_119_040
    assert 4 * 1152 == 4608
    # the near alternatives do not fit: norm over the merged 4608, or no norm, or bias-free Linears
    h = 4608
    assert 2 * h + (h * h + h) + (h * 4096 + 4096) != 40_119_040
    assert (h * h + h) + (h * 4096 + 4096) != 40_119_040
    assert 2 * 1152 + h * h + h * 4096 != 40_119_040


def test_layer_norm_closed_forms():
    rng = np.random.default_rng(11)
    x = rng.normal(size=(5, 40)) * 3 + 2
    y = O.layer_norm(x, np.ones(40), np.zeros(40), eps=0.0)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(y.var(axis=1), 1, rtol=1e-12)
    b = rng.normal(size=40)
    np.testing.assert_allclose(O.layer_norm(np.full((2, 40), 3.5), rng.normal(size=40), b), np.stack([b, b]), atol=1e-12)
    # hand value: row (1, 3): mean 2, var 1 -> (-1, 1) / sqrt(1 + eps)
    np.testing.assert_allclose(O.layer_norm(np.array([[1.0, 3.0]]), np.array([2.0, 1.0]), np.array([0.5, 0.0]), 0.0),
                               [[-1.5, 1.0]], atol=1e-15)


def test_gelu_values():
    np.testing.assert_allclose(O.gelu(np.array([0.0, 1.0, -1.0])), [0.0, 0.8413447460685429, -0.15865525393145707],
                               rtol=1e-15, atol=1e-16)
    z = np.linspace(-6, 6, 61)
    np.testing.assert_allclose(O.gelu(z) - O.gelu(-z), z, atol=1e-13)     # z Phi(z) - (-z) Phi(-z) = z
    np.testing.assert_allclose(O.gelu(np.array([10.0])), [10.0], rtol=1e-15)


def test_patch_merger_composition_and_padding():
    rng = np.random.default_rng(12)
    d, r, e = 3, 2, 5
    grids = [(3, 5), (2, 2)]
    x = rng.normal(size=(15 + 4, d))
    lw, lb = 1 + 0.1 * rng.normal(size=d), 0.1 * rng.normal(size=d)
    w1, b1 = rng.normal(size=(4 * d, 4 * d)), rng.normal(size=4 * d)
    w2, b2 = rng.normal(size=(e, 4 * d)), rng.normal(size=e)
    out, cu = O.patch_merger(x, grids, r, lw, lb, w1, b1, w2, b2)
    assert out.shape == (6 + 1, e) and list(cu) == [0, 6, 7]
    # written out step by step for token (0, 2) of image 0: patches (0,4), (1,4) and two padding slots
    xn = O.layer_norm(x, lw, lb)
    m = np.concatenate([xn[4], np.zeros(d), xn[5 + 4], np.zeros(d)])
    np.testing.assert_allclose(out[2], O.gelu(w1 @ m + b1) @ w2.T + b2, rtol=1e-12, atol=1e-12)
    # identity-like first layer: w1 = I, b1 = 0 gives w2 . gelu(merged) + b2
    out_i, _ = O.patch_merger(x, grids, r, lw, lb, np.eye(4 * d), np.zeros(4 * d), w2, b2)
    merged, _ = O.aligner_merge(xn, grids, r)
    np.testing.assert_allclose(out_i, O.gelu(merged) @ w2.T + b2, rtol=1e-12, atol=1e-12)



# ------------------------------------------------------------------------ image-token bridge
def _golden_rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_image_layout_hand_table_and_length():
    # hand-written layout of a 3x5 grid at r = 2; catches a missing newline, a swapped
    # start/end or a token row of the wrong width.
    want = [int(v) for v in _golden_rows("image_layout_3x5_r2.txt")[0]]
    assert O.image_layout(3, 5, 2).tolist() == want
    # closed form: 2 + g_h (g_w + 1) entries, g_h g_w of them features; the pages' grids.
    for n_h, n_w in [(28, 28), (27, 37), (37, 27), (10, 78), (112, 7), (1, 1)]:
        for r in (1, 2, 3):
            g_h, g_w = -(-n_h // r), -(-n_w // r)
            lay = O.image_layout(n_h, n_w, r)
            assert len(lay) == 2 + g_h * (g_w + 1)
            assert int((lay == O.TOK_IMAGE).sum()) == g_h * g_w
            assert int((lay == O.TOK_NEWLINE).sum()) == g_h
            # each newline closes a row: it sits g_w + 1 after the previous one
            nl = np.flatnonzero(lay == O.TOK_NEWLINE)
            assert (np.diff(np.concatenate([[0], nl])) == g_w + 1).all()


def _bridge_case():
    # two sequences of 24 holding three images (3x5 -> 6 tokens, 1x1 -> 1, 4x4 -> 4 at r = 2)
    # with text around and between them, and one image_pad inside the last span.
    lay = [O.image_layout(3, 5, 2), O.image_layout(1, 1, 2), O.image_layout(4, 4, 2)]
    last = np.concatenate([lay[2][:-1], [O.TOK_PAD], lay[2][-1:]])
    s0 = np.concatenate([[-1, -1], lay[0], [-1], lay[1], [-1] * 7])
    s1 = np.concatenate([[-1] * 3, last, [-1] * 12])
    assert len(s0) == 24 and len(s1) == 24
    return np.stack([s0, s1]).astype(np.int32), [6, 1, 4]


def test_merge_image_embeddings_encoded_rows():
    # rows carry their own identity: text rows 1000 + position, token k -> k, sentinel i ->
    # -(i + 1).  Catches a wrong token order, a skipped or repeated token, a sentinel mix-up and
    # a text row that is touched.
    types, per_image = _bridge_case()
    b, s = types.shape
    e = 3
    embeds = (1000.0 + np.arange(b * s, dtype=np.float64)).repeat(e).reshape(b, s, e)
    toks = np.arange(sum(per_image), dtype=np.float64).repeat(e).reshape(-1, e)
    sent = -(1.0 + np.arange(4, dtype=np.float64)).repeat(e).reshape(4, e)
    out = O.merge_image_embeddings(embeds, types, toks, sent, per_image)
    flat_t, flat_o, flat_in = types.reshape(-1), out.reshape(-1, e), embeds.reshape(-1, e)
    feats = flat_o[flat_t == O.TOK_IMAGE, 0]
    assert feats.tolist() == list(range(sum(per_image)))
    # the sentinel rows are image_start, image_end, image_newline, image_pad (types 1, 2, 3, 4),
    # written out here rather than read from the oracle
    for code, row in ((1, 0), (2, 1), (3, 2), (4, 3)):
        assert (flat_o[flat_t == code] == -(row + 1.0)).all()
    np.testing.assert_array_equal(flat_o[flat_t == O.TOK_TEXT], flat_in[flat_t == O.TOK_TEXT])
    assert int((flat_t == O.TOK_PAD).sum()) == 1


@pytest.mark.parametrize("mutate", ["drop_feature", "extra_feature", "open_span", "stray_pad",
                                    "nested_start", "bad_code", "few_images", "text_in_span"])
def test_merge_image_embeddings_rejects_layouts_that_do_not_fit(mutate):
    types, per_image = _bridge_case()
    t = types.copy()
    f0 = int(np.flatnonzero(t[0] == O.TOK_IMAGE)[0])
    if mutate == "drop_feature":
        t[0, f0] = O.TOK_PAD
    elif mutate == "extra_feature":
        t[1, int(np.flatnonzero(t[1] == O.TOK_PAD)[0])] = O.TOK_IMAGE
    elif mutate == "open_span":
        t[1, int(np.flatnonzero(t[1] == O.TOK_END)[0])] = O.TOK_NEWLINE
    elif mutate == "stray_pad":
        t[0, 0] = O.TOK_PAD
    elif mutate == "nested_start":
        t[0, f0] = O.TOK_START
    elif mutate == "bad_code":
        t[0, 0] = 7
    elif mutate == "few_images":
        per_image = per_image + [1]
    elif mutate == "text_in_span":  # feature counts intact, one newline turned into text
        t[0, int(np.flatnonzero(t[0] == O.TOK_NEWLINE)[0])] = O.TOK_TEXT
    z = np.zeros(t.shape + (2,))
    with pytest.raises(ValueError):
        O.merge_image_embeddings(z, t, np.zeros((sum(per_image), 2)), np.zeros((4, 2)), per_image)


@pytest.mark.parametrize("row", [[1, 0, -1, 0, 2],      # text inside a span
                                 [1, 0, 1, 0, 2, 2],    # a start inside an open span
                                 [0, 1, 0, 2],          # a feature before any span
                                 [1, 0, 3],             # a span never closed
                                 [2, 1, 0, 2],          # an end outside a span
                                 [1, 5, 2]])            # an unknown code
def test_image_spans_rejects_malformed_rows(row):
    with pytest.raises(ValueError):
        O.image_spans(np.array(row))
    with pytest.raises(ValueError):
        O.image_visibility(np.zeros((1, len(row), len(row))), np.array([row]))


def test_image_visibility_hand_table():
    rows = _golden_rows("image_visibility_12.txt")
    types = np.array([[int(v) for v in rows[0]]])
    n = types.shape[1]
    causal = np.where(np.arange(n)[None, :] > np.arange(n)[:, None], -np.inf, 0.0)[None]
    want = np.array([[0.0 if c == "." else -np.inf for c in row] for row in rows[1:]])
    np.testing.assert_array_equal(O.image_visibility(causal, types)[0], want)
    assert O.image_spans(types[0]) == [(2, 6), (8, 11)]


def test_image_visibility_keeps_text_and_other_samples():
    # random additive mask: entries outside the spans are untouched, the spans' blocks are 0,
    # and a sample without images is unchanged; catches a span leaking across samples.
    types, _ = _bridge_case()
    types = np.concatenate([types, np.full((1, types.shape[1]), -1, np.int32)])
    m = RNG.normal(size=(3, 24, 24))
    out = O.image_visibility(m, types)
    inside = np.zeros_like(m, dtype=bool)
    for b in range(3):
        for a, e in O.image_spans(types[b]):
            inside[b, a:e + 1, a:e + 1] = True
    assert inside[0].sum() == 10 ** 2 + 4 ** 2 and inside[1].sum() == 9 ** 2 and not inside[2].any()
    assert (out[inside] == 0).all()
    np.testing.assert_array_equal(out[~inside], m[~inside])

"""Pins of the fp64 backward oracle (oracle/dsv4v_grad.py) to facts other than itself: central
finite differences of the forward oracle, closed forms and invariants.  CPU only.

Each gradient is the gradient of L = sum(f(inputs) * d_out).  A finite-difference check perturbs
one input along a random direction u and compares (L(+h u) - L(-h u)) / 2h with <grad, u>; in
float64 with h = 1e-5 both agree to ~1e-9 relative, while a dropped term, a wrong sign, a
transposed operand or a wrong scale is off by O(1)."""
import math

import numpy as np
import pytest

from oracle import dsv4v_grad as G
from oracle import dsv4v_oracle as O

RNG = np.random.default_rng(2024)
D, H, F = 16, 2, 24  # head_dim 8: the rotary table has two frequencies per axis
GRIDS = [(2, 3), (1, 2), (3, 1)]
P = sum(h * w for h, w in GRIDS)


def directional_fd(loss, value, grad, n_dirs=3, h=1e-5):
    """Checks <grad, u> against the central difference of loss along random directions u."""
    for _ in range(n_dirs):
        u = RNG.normal(size=value.shape)
        fd = (loss(value + h * u) - loss(value - h * u)) / (2 * h)
        an = float(np.sum(grad * u))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (fd, an)


def layer(scale=0.3):
    return {"norm1_w": 1 + 0.1 * RNG.normal(size=D), "wqkv": scale * RNG.normal(size=(3 * D, D)),
            "wo": scale * RNG.normal(size=(D, D)), "norm2_w": 1 + 0.1 * RNG.normal(size=D),
            "w_gate": scale * RNG.normal(size=(F, D)), "w_up": scale * RNG.normal(size=(F, D)),
            "w_down": scale * RNG.normal(size=(D, F))}


def tables():
    return O.packed_cos_sin(GRIDS, D // H // 2, 100.0)


# ------------------------------------------------------------------------------- RMSNorm
def test_rmsnorm_backward_elementwise_fd():
    x, w, dy = RNG.normal(size=(3, 7)), RNG.normal(size=7), RNG.normal(size=(3, 7))
    dx, dw = G.rmsnorm_backward(x, w, dy, 1e-3)
    h = 1e-6
    for idx in np.ndindex(x.shape):
        e = np.zeros_like(x)
        e[idx] = h
        fd = (np.sum(O.rmsnorm(x + e, w, 1e-3) * dy) - np.sum(O.rmsnorm(x - e, w, 1e-3) * dy)) / (2 * h)
        assert abs(fd - dx[idx]) < 1e-8
    for i in range(7):
        e = np.zeros(7)
        e[i] = h
        fd = (np.sum(O.rmsnorm(x, w + e, 1e-3) * dy) - np.sum(O.rmsnorm(x, w - e, 1e-3) * dy)) / (2 * h)
        assert abs(fd - dw[i]) < 1e-8


def test_rmsnorm_backward_scale_invariance():
    # with eps = 0 the norm is invariant to scaling x, so the gradient is orthogonal to x per row
    x, w, dy = RNG.normal(size=(4, 9)), RNG.normal(size=9), RNG.normal(size=(4, 9))
    dx, _ = G.rmsnorm_backward(x, w, dy, 0.0)
    np.testing.assert_allclose(np.sum(dx * x, axis=1), 0.0, atol=1e-12)


# ------------------------------------------------------------------------------- rotation
def test_rotary_backward_is_the_inverse_rotation():
    # the rotation is orthogonal: its transpose undoes it and keeps norms
    cos, sin = tables()
    x = RNG.normal(size=(P, H, D // H))
    np.testing.assert_allclose(G.rotary_backward(O.apply_vision_rotary(x, cos, sin), cos, sin), x, atol=1e-13)
    d = RNG.normal(size=x.shape)
    np.testing.assert_allclose(np.linalg.norm(G.rotary_backward(d, cos, sin)), np.linalg.norm(d), rtol=1e-13)


def test_rotary_backward_fd():
    cos, sin = tables()
    x, d = RNG.normal(size=(P, H, D // H)), RNG.normal(size=(P, H, D // H))
    directional_fd(lambda v: np.sum(O.apply_vision_rotary(v, cos, sin) * d), x, G.rotary_backward(d, cos, sin))


# ------------------------------------------------------------------------------ attention
def test_attention_backward_fd():
    q, k, v = (RNG.normal(size=(P, H, D // H)) for _ in range(3))
    do = RNG.normal(size=(P, D))
    dq, dk, dv = G.attention_backward(q, k, v, do, GRIDS)
    directional_fd(lambda t: np.sum(O.attention_packed(t, k, v, GRIDS) * do), q, dq)
    directional_fd(lambda t: np.sum(O.attention_packed(q, t, v, GRIDS) * do), k, dk)
    directional_fd(lambda t: np.sum(O.attention_packed(q, k, t, GRIDS) * do), v, dv)


def test_attention_backward_closed_forms():
    n, hd = 6, 8
    q, k, do = RNG.normal(size=(n, hd)), RNG.normal(size=(n, hd)), RNG.normal(size=(n, hd))
    # identical value rows: the output does not depend on q or k
    v = np.tile(RNG.normal(size=hd), (n, 1))
    dq, dk, _ = G.attention_backward_one_head(q, k, v, do)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    np.testing.assert_allclose(dk, 0.0, atol=1e-13)
    # identical key rows: uniform attention whatever q is, so dq = 0 (softmax rows of dS sum to 0)
    v = RNG.normal(size=(n, hd))
    dq, _, dv = G.attention_backward_one_head(q, np.tile(k[0], (n, 1)), v, do)
    np.testing.assert_allclose(dq, 0.0, atol=1e-13)
    np.testing.assert_allclose(dv, np.tile(do.mean(axis=0), (n, 1)), atol=1e-13)  # P = 1/n everywhere
    # the probabilities sum to one per query, so the value gradients sum to the output gradients
    _, _, dv = G.attention_backward_one_head(q, k, v, do)
    np.testing.assert_allclose(dv.sum(axis=0), do.sum(axis=0), atol=1e-12)


def test_attention_backward_isolates_images():
    q, k, v = (RNG.normal(size=(P, H, D // H)) for _ in range(3))
    do = RNG.normal(size=(P, D))
    do[:6] = 0.0  # no gradient on the first image's outputs
    dq, dk, dv = G.attention_backward(q, k, v, do, GRIDS)
    assert not dq[:6].any() and not dk[:6].any() and not dv[:6].any()


# ------------------------------------------------------------------------------- SwiGLU
def test_silu_grad_values():
    assert G.silu_grad(0.0) == 0.5
    np.testing.assert_allclose(G.silu_grad([40.0, -40.0]), [1.0, 0.0], atol=1e-15)
    z = RNG.normal(size=20) * 3
    np.testing.assert_allclose(G.silu_grad(z), (O.silu(z + 1e-6) - O.silu(z - 1e-6)) / 2e-6, atol=1e-9)


def test_mlp_backward_fd():
    lw = layer()
    y, do = RNG.normal(size=(P, D)), RNG.normal(size=(P, D))
    dy, dwg, dwu, dwd = G.mlp_backward(y, lw["w_gate"], lw["w_up"], lw["w_down"], do)
    f = lambda y_, g_, u_, d_: np.sum(O.mlp(y_, g_, u_, d_) * do)
    directional_fd(lambda t: f(t, lw["w_gate"], lw["w_up"], lw["w_down"]), y, dy)
    directional_fd(lambda t: f(y, t, lw["w_up"], lw["w_down"]), lw["w_gate"], dwg)
    directional_fd(lambda t: f(y, lw["w_gate"], t, lw["w_down"]), lw["w_up"], dwu)
    directional_fd(lambda t: f(y, lw["w_gate"], lw["w_up"], t), lw["w_down"], dwd)


def test_mlp_backward_gate_up_not_swapped():
    # scalar case: out = silu(g y) (u y) d; d out / d g = y silu'(g y) (u y) d, not silu(u y) ...
    y, g, u, d = np.array([[0.7]]), np.array([[1.3]]), np.array([[-0.4]]), np.array([[2.0]])
    _, dwg, dwu, dwd = G.mlp_backward(y, g, u, d, np.ones((1, 1)))
    z = 1.3 * 0.7
    assert math.isclose(dwg[0, 0], 0.7 * float(G.silu_grad(z)) * (-0.4 * 0.7) * 2.0, rel_tol=1e-14)
    assert math.isclose(dwu[0, 0], 0.7 * float(O.silu(z)) * 2.0, rel_tol=1e-14)
    assert math.isclose(dwd[0, 0], float(O.silu(z)) * (-0.4 * 0.7), rel_tol=1e-14)


# ------------------------------------------------------------------- projection + rotation
def test_qkv_rope_backward_fd():
    cos, sin = tables()
    w = 0.3 * RNG.normal(size=(3 * D, D))
    y = RNG.normal(size=(P, D))
    dq, dk, dv = (RNG.normal(size=(P, H, D // H)) for _ in range(3))

    def loss(y_, w_):
        q, k, v = O.qkv_rope(y_, w_, cos, sin, H)
        return np.sum(q * dq) + np.sum(k * dk) + np.sum(v * dv)

    dy, dw = G.qkv_rope_backward(y, w, cos, sin, H, dq, dk, dv)
    directional_fd(lambda t: loss(t, w), y, dy)
    directional_fd(lambda t: loss(y, t), w, dw)


# --------------------------------------------------------------------------------- block
def test_block_backward_fd_every_input():
    cos, sin = tables()
    lw = layer()
    x, do = RNG.normal(size=(P, D)), RNG.normal(size=(P, D))
    dx, grads = G.block_backward(x, lw, cos, sin, GRIDS, H, do)
    loss = lambda x_, l_: np.sum(O.block_forward(x_, l_, cos, sin, GRIDS, H) * do)
    directional_fd(lambda t: loss(t, lw), x, dx)
    for key in lw:
        directional_fd(lambda t: loss(x, {**lw, key: t}), lw[key], grads[key], n_dirs=2)


def test_block_backward_identity_when_projections_vanish():
    # wo = 0 and w_down = 0 make the block the identity: dx = d_out and no gradient reaches
    # the projection in front of attention or the norm scales
    cos, sin = tables()
    lw = {**layer(), "wo": np.zeros((D, D)), "w_down": np.zeros((D, F))}
    x, do = RNG.normal(size=(P, D)), RNG.normal(size=(P, D))
    dx, grads = G.block_backward(x, lw, cos, sin, GRIDS, H, do)
    np.testing.assert_array_equal(dx, do)
    for key in ("wqkv", "norm1_w", "norm2_w", "w_gate", "w_up"):
        assert not grads[key].any(), key
    assert grads["wo"].any() and grads["w_down"].any()


def test_block_backward_isolates_images():
    cos, sin = tables()
    lw = layer()
    x, do = RNG.normal(size=(P, D)), RNG.normal(size=(P, D))
    do[6:] = 0.0  # gradient only on the first image
    dx, _ = G.block_backward(x, lw, cos, sin, GRIDS, H, do)
    assert not dx[6:].any()


# --------------------------------------------------------------------------------- tower
def test_tower_backward_fd():
    layers = [layer(0.2), layer(0.2)]
    fn = 1 + 0.1 * RNG.normal(size=D)
    x, do = RNG.normal(size=(P, D)), RNG.normal(size=(P, D))
    dx, grads, dfn = G.tower_backward(x, layers, fn, GRIDS, H, do, rope_theta=100.0)
    loss = lambda x_, ls, f_: np.sum(O.tower_forward(x_, ls, f_, GRIDS, H, 100.0) * do)
    directional_fd(lambda t: loss(t, layers, fn), x, dx)
    directional_fd(lambda t: loss(x, layers, t), fn, dfn)
    directional_fd(lambda t: loss(x, [{**layers[0], "wqkv": t}, layers[1]], fn), layers[0]["wqkv"],
                   grads[0]["wqkv"], n_dirs=2)
    directional_fd(lambda t: loss(x, [layers[0], {**layers[1], "w_up": t}], fn), layers[1]["w_up"],
                   grads[1]["w_up"], n_dirs=2)
    _, _, none = G.tower_backward(x, layers, None, GRIDS, H, do, rope_theta=100.0)
    assert none is None

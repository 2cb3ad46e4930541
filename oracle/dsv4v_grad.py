"""fp64 CPU oracle of the gradients of the vision tower (the backward of the forward oracle).

TEST INFRASTRUCTURE ONLY, like dsv4v_oracle (which it builds on): only the tests may import it.
The pages train the tower and test "ragged grids and backward" ([PR], Validation) but print no
backward; every function here is the chain rule applied by hand to the forward definitions of
dsv4v_oracle, one step at a time, in float64, with numpy's matmul as the only library primitive.
Each function returns the gradient of sum(out * d_out) with respect to its inputs and weights;
the not-gpu tests pin every one of them against central finite differences and closed forms.

Layouts follow dsv4v_oracle: packed activations [P, D], weights [out, in], grids (n_h, n_w).
"""
from __future__ import annotations

import math

import numpy as np

from oracle import dsv4v_oracle as O


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def rmsnorm_backward(x, weight, d_out, eps: float = 1e-6):
    """y = w * x * r with r = 1 / sqrt(mean(x^2) + eps).  With g = d_out * w:
    dx = r g - x r^3 (g . x) / D, dw = sum over rows of d_out * x * r."""
    x, w, dy = _f64(x), _f64(weight), _f64(d_out)
    d = x.shape[-1]
    r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    g = dy * w
    dx = r * g - x * r ** 3 * np.sum(g * x, axis=-1, keepdims=True) / d
    dw = np.sum(dy * x * r, axis=0)
    return dx, dw


def rotary_backward(d_out, cos, sin) -> np.ndarray:
    """The rotation is orthogonal, so its transpose is the rotation by the negative angle:
    with out = (a c - b s, b c + a s), da = d1 c + d2 s and db = d2 c - d1 s."""
    d = _f64(d_out)
    half = d.shape[-1] // 2
    c = _f64(cos)[:, None, :]
    s = _f64(sin)[:, None, :]
    d1, d2 = d[..., :half], d[..., half:]
    return np.concatenate([d1 * c + d2 * s, d2 * c - d1 * s], axis=-1)


def attention_backward_one_head(q, k, v, d_out):
    """o = P v with P = softmax(q k^T / sqrt(hd)) row-wise, for one image and one head.
    dv = P^T do; dP = do v^T; dS = P * (dP - rowsum(dP * P)); dq = dS k / sqrt(hd);
    dk = dS^T q / sqrt(hd)."""
    q, k, v, do = _f64(q), _f64(k), _f64(v), _f64(d_out)
    scale = 1.0 / math.sqrt(q.shape[-1])
    p = O.attention_probs(q, k)
    dv = p.T @ do
    dp = do @ v.T
    ds = p * (dp - np.sum(dp * p, axis=1, keepdims=True))
    return ds @ k * scale, ds.T @ q * scale, dv


def attention_backward(q, k, v, d_out, grids):
    """Packed attention ([P, H, hd] each, output [P, H*hd]): every image and head on its own."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    n_heads, hd = q.shape[1], q.shape[2]
    do = _f64(d_out).reshape(-1, n_heads, hd)
    dq, dk, dv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    cu = O.cu_from_grids(grids)
    for a, b in zip(cu[:-1], cu[1:]):
        for h in range(n_heads):
            dq[a:b, h], dk[a:b, h], dv[a:b, h] = attention_backward_one_head(q[a:b, h], k[a:b, h], v[a:b, h],
                                                                             do[a:b, h])
    return dq, dk, dv


def silu_grad(z) -> np.ndarray:
    """d silu / dz = sigma(z) (1 + z (1 - sigma(z)))."""
    z = _f64(z)
    sg = 1.0 / (1.0 + np.exp(-z))
    return sg * (1.0 + z * (1.0 - sg))


def mlp_backward(y, w_gate, w_up, w_down, d_out):
    """out = (silu(g) * u) Wd^T with g = y Wg^T, u = y Wu^T.  Returns dy and the weight
    gradients (dWg, dWu, dWd)."""
    y, wg, wu, wd, do = _f64(y), _f64(w_gate), _f64(w_up), _f64(w_down), _f64(d_out)
    g, u = y @ wg.T, y @ wu.T
    h = O.silu(g) * u
    dwd = do.T @ h
    dh = do @ wd
    dg = dh * u * silu_grad(g)
    du = dh * O.silu(g)
    return dg @ wg + du @ wu, dg.T @ y, du.T @ y, dwd


def qkv_rope_backward(y, wqkv, cos, sin, n_heads: int, dq, dk, dv):
    """Back through the rotation of q and k, then the fused projection.  Returns dy, dWqkv."""
    y, w = _f64(y), _f64(wqkv)
    p = y.shape[0]
    dqkv = np.concatenate([rotary_backward(dq, cos, sin).reshape(p, -1),
                           rotary_backward(dk, cos, sin).reshape(p, -1), _f64(dv).reshape(p, -1)], axis=1)
    return dqkv @ w, dqkv.T @ y


def block_backward(x, layer: dict, cos, sin, grids, n_heads: int, d_out, eps: float = 1e-6):
    """Gradient of sum(block_forward(x) * d_out): recomputes the forward's intermediates, then
    walks back through the MLP branch, norm2, the output projection, attention, the projection
    and rotation, and norm1.  Returns dx and a dict of weight gradients keyed like `layer`."""
    x, do = _f64(x), _f64(d_out)
    wo = _f64(layer["wo"])
    y1 = O.rmsnorm(x, layer["norm1_w"], eps)
    q, k, v = O.qkv_rope(y1, layer["wqkv"], cos, sin, n_heads)
    att = O.attention_packed(q, k, v, grids)
    x2 = x + att @ wo.T
    y2 = O.rmsnorm(x2, layer["norm2_w"], eps)

    dy2, dwg, dwu, dwd = mlp_backward(y2, layer["w_gate"], layer["w_up"], layer["w_down"], do)
    dx2_norm, dn2 = rmsnorm_backward(x2, layer["norm2_w"], dy2, eps)
    dx2 = do + dx2_norm
    dwo = dx2.T @ att
    datt = dx2 @ wo
    dq, dk, dv = attention_backward(q, k, v, datt, grids)
    dy1, dwqkv = qkv_rope_backward(y1, layer["wqkv"], cos, sin, n_heads, dq, dk, dv)
    dx_norm, dn1 = rmsnorm_backward(x, layer["norm1_w"], dy1, eps)
    grads = {"norm1_w": dn1, "wqkv": dwqkv, "wo": dwo, "norm2_w": dn2, "w_gate": dwg, "w_up": dwu,
             "w_down": dwd}
    return dx2 + dx_norm, grads


def tower_backward(x, layers, final_norm_w, grids, n_heads: int, d_out, rope_theta: float = 10000.0,
                   eps: float = 1e-6):
    """Gradient of sum(tower_forward(x) * d_out): the forward is run once to keep every block's
    input, then the final norm and the blocks are walked in reverse.  Returns dx, the list of
    per-layer gradient dicts, and the final norm's weight gradient (None without a final norm)."""
    x = _f64(x)
    hd = x.shape[1] // n_heads
    cos, sin = O.packed_cos_sin(grids, hd // 2, rope_theta)
    inputs = []
    for layer in layers:
        inputs.append(x)
        x = O.block_forward(x, layer, cos, sin, grids, n_heads, eps)
    d = _f64(d_out)
    d_final = None
    if final_norm_w is not None:
        d, d_final = rmsnorm_backward(x, final_norm_w, d, eps)
    grads = [None] * len(layers)
    for i in reversed(range(len(layers))):
        d, grads[i] = block_backward(inputs[i], layers[i], cos, sin, grids, n_heads, d, eps)
    return d, grads, d_final

"""Parity of the backward calls with the fp64 backward oracle (oracle/dsv4v_grad.py), through the
C ABI.

Tolerances.  The inputs are bf16 values, which the oracle widens exactly.  The kernels compute in
fp32 and store every activation and gradient in bf16, one rounding (<= 2^-9 relative) per stored
tensor.
  * Attention backward: three bf16 inputs and one bf16 output, so rel. Frobenius <= 1e-2.
  * RMSNorm backward: dx is within 2^-8 |ref| + 1e-3 element by element; dw (an fp32 sum over
    the rows) has rel. Frobenius <= 1e-4.
  * Block and tower backward: about a dozen bf16 roundings chained through the recompute and the
    backward, like the forward tower, so rel. Frobenius <= 3e-2.  dx is compared after removing
    the residual term d_out, which would otherwise hide errors in the branches."""
import numpy as np
import pytest
import torch

from gpu_util import dev, f32, random_bf16, rel_fro, to_np
from oracle import dsv4v_grad as G
from oracle import dsv4v_oracle as O
from vision_transformer_encoder_dsv4v_b200 import dsv4v as A

pytestmark = pytest.mark.gpu

D, H, F = 1024, 16, 2816
GRIDS = {
    "28x28": [(28, 28)],
    "ragged4": [(27, 37), (37, 27), (10, 78), (112, 7)],
    "small": [(3, 5), (1, 1), (9, 14)],
    "one_patch": [(1, 1)],  # the weight gradients reduce over K = P = 1
}


def cfg_bf16(n_layers=1):
    return A.make_config(D, H, F, 2, 4096, n_layers, 1e-6, 10000.0, A.DSV4V_BF16)


def bwd_ws(cfg, b):
    n = A.dsv4v_backward_workspace_size(cfg, b)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def random_layer(seed):
    rng = np.random.default_rng(seed)
    t = {"wqkv": random_bf16((3 * D, D), 0.02, seed + 1), "wo": random_bf16((D, D), 0.02, seed + 2),
         "w_gate": random_bf16((F, D), 0.02, seed + 3), "w_up": random_bf16((F, D), 0.02, seed + 4),
         "w_down": random_bf16((D, F), 0.02, seed + 5)}
    norms = {"norm1_w": (1 + 0.1 * rng.standard_normal(D)).astype(np.float32),
             "norm2_w": (1 + 0.1 * rng.standard_normal(D)).astype(np.float32)}
    host = {k: v.values for k, v in t.items()}
    host.update(norms)
    device = {k: dev(v) for k, v in t.items()}
    device.update({k: f32(v) for k, v in norms.items()})
    return host, device


def grad_buffers():
    g = {"norm1_w": torch.empty(D, device="cuda"), "norm2_w": torch.empty(D, device="cuda"),
         "wqkv": torch.empty(3 * D, D, dtype=torch.bfloat16, device="cuda"),
         "wo": torch.empty(D, D, dtype=torch.bfloat16, device="cuda"),
         "w_gate": torch.empty(F, D, dtype=torch.bfloat16, device="cuda"),
         "w_up": torch.empty(F, D, dtype=torch.bfloat16, device="cuda"),
         "w_down": torch.empty(D, F, dtype=torch.bfloat16, device="cuda")}
    return g, A.block_grads(g["norm1_w"], g["norm2_w"], g["wqkv"], g["wo"], g["w_gate"], g["w_up"], g["w_down"])


def tables(cfg, b):
    cos = torch.empty(b.n_patches, D // H // 2, device="cuda")
    sin = torch.empty_like(cos)
    A.dsv4v_rope2d_table(cfg, b, cos, sin)
    return cos, sin


@pytest.mark.parametrize("name", list(GRIDS) + ["lines"])
def test_attention_backward(name):
    grids = GRIDS.get(name, [(1, 37), (37, 1), (2, 2)])
    cfg = cfg_bf16()
    b = A.BatchRef(grids)
    P = b.n_patches
    qkv = random_bf16((P, 3 * D), 1.0, seed=P)
    do = random_bf16((P, D), 1.0, seed=P + 1)
    qkv_d = dev(qkv)
    out = torch.empty(P, D, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_attention(cfg, b, qkv_d, out)
    dqkv = torch.empty(P, 3 * D, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_attention_backward(cfg, b, qkv_d, out, dev(do), dqkv, bwd_ws(cfg, b))
    assert A.dsv4v_device_error() == 0
    q, k, v = (qkv.values[:, i * D:(i + 1) * D].reshape(P, H, D // H) for i in range(3))
    dq, dk, dv = G.attention_backward(q, k, v, do.values, grids)
    got = to_np(dqkv)
    for i, want in enumerate((dq, dk, dv)):
        w, g = want.reshape(P, D), got[:, i * D:(i + 1) * D]
        if not w.any():  # one key: the softmax is exactly 1, so dq = dk = 0 up to fp32 rounding
            assert np.linalg.norm(g) <= 1e-3 * np.linalg.norm(do.values), i
            continue
        err = rel_fro(g, w)
        assert err < 1e-2, (i, err)


@pytest.mark.parametrize("name", ["28x28", "small", "one_patch"])
def test_rmsnorm_backward(name):
    cfg = cfg_bf16()
    b = A.BatchRef(GRIDS[name])
    P = b.n_patches
    x = random_bf16((P, D), 2.0, seed=3)
    dy = random_bf16((P, D), 1.0, seed=4)
    d_in = random_bf16((P, D), 1.0, seed=5)
    w = (1 + 0.1 * np.random.default_rng(6).standard_normal(D)).astype(np.float32)
    dx = torch.empty(P, D, dtype=torch.bfloat16, device="cuda")
    dw = torch.empty(D, device="cuda")
    A.dsv4v_rmsnorm_backward(cfg, b, dev(x), f32(w), dev(dy), dev(d_in), dx, dw, bwd_ws(cfg, b))
    want_dx, want_dw = G.rmsnorm_backward(x.values, w, dy.values, 1e-6)
    want_dx = want_dx + d_in.values
    got = to_np(dx)
    assert (np.abs(got - want_dx) <= 2.0 ** -8 * np.abs(want_dx) + 1e-3).all()
    assert rel_fro(dw.cpu().numpy(), want_dw) < 1e-4


@pytest.mark.parametrize("name", list(GRIDS))
def test_block_backward(name):
    grids = GRIDS[name]
    cfg = cfg_bf16()
    b = A.BatchRef(grids)
    P = b.n_patches
    host, device = random_layer(11)
    x = random_bf16((P, D), 1.0, seed=12)
    do = random_bf16((P, D), 1.0, seed=13)
    cos, sin = tables(cfg, b)
    dx = torch.empty(P, D, dtype=torch.bfloat16, device="cuda")
    g, grads = grad_buffers()
    A.dsv4v_block_backward(cfg, b, A.block_weights(device), cos, sin, dev(x), dev(do), dx, grads, bwd_ws(cfg, b))
    assert A.dsv4v_device_error() == 0
    c_o, s_o = O.packed_cos_sin(grids, D // H // 2, 10000.0)
    want_dx, want = G.block_backward(x.values, host, c_o, s_o, grids, H, do.values)
    assert rel_fro(to_np(dx) - do.values, want_dx - do.values) < 3e-2
    for key, t in g.items():
        err = rel_fro(to_np(t), want[key])
        assert err < 3e-2, (key, err)


def test_tower_backward_two_layers():
    grids = GRIDS["small"]
    cfg = cfg_bf16(n_layers=2)
    b = A.BatchRef(grids)
    P = b.n_patches
    layers = [random_layer(21), random_layer(31)]
    fn = (1 + 0.1 * np.random.default_rng(41).standard_normal(D)).astype(np.float32)
    x = random_bf16((P, D), 1.0, seed=42)
    do = random_bf16((P, D), 1.0, seed=43)
    cos, sin = tables(cfg, b)
    # the forward on the GPU keeps each block's input and the last block's output
    ws_f = torch.empty(A.dsv4v_workspace_size(cfg, b), dtype=torch.uint8, device="cuda")
    inputs = [dev(x)]
    cur = inputs[0].clone()
    for _, d in layers:
        A.dsv4v_block_forward(cfg, b, A.block_weights(d), cos, sin, cur, ws_f)
        inputs.append(cur.clone())
    x_last = inputs.pop()
    bufs = [grad_buffers() for _ in layers]
    dx = torch.empty(P, D, dtype=torch.bfloat16, device="cuda")
    dfn = torch.empty(D, device="cuda")
    A.dsv4v_tower_backward(cfg, b, [A.block_weights(d) for _, d in layers], f32(fn), inputs, x_last, dev(do), dx,
                           [gr for _, gr in bufs], dfn, bwd_ws(cfg, b))
    assert A.dsv4v_device_error() == 0
    want_dx, want, want_fn = G.tower_backward(x.values, [h for h, _ in layers], fn, grids, H, do.values)
    assert rel_fro(to_np(dx), want_dx) < 3e-2
    assert rel_fro(dfn.cpu().numpy(), want_fn) < 3e-2
    for (g, _), w in zip(bufs, want):
        for key, t in g.items():
            err = rel_fro(to_np(t), w[key])
            assert err < 3e-2, (key, err)


def test_backward_rejects_fp32_config():
    cfg = A.make_config(64, 4, 128, 2, 128, 1, 1e-6, 10000.0, A.DSV4V_F32)
    b = A.BatchRef([(3, 5)])
    assert A.dsv4v_backward_workspace_size(cfg, b) == 0
    with pytest.raises(A.Dsv4vError) as e:
        A.dsv4v_attention_backward(cfg, b, None, None, None, None, None)
    assert e.value.status == 2

"""Helpers shared by the GPU tests: upload seeded inputs, run the library through its C ABI,
compare against the oracle."""
import numpy as np
import torch

from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
from vision_transformer_encoder_dsv4v_b200 import synth


def dev(t: "synth.Tensor", device="cuda"):
    """A stored input on the device in its storage dtype (bf16 from its raw bits, else fp32)."""
    if t.bits is not None:
        return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(t.values)).to(device)


def f32(a, device="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def to_np(t):
    return t.float().cpu().numpy().astype(np.float64)


def config_of(wl: "synth.Workload", n_layers=None):
    return A.make_config(wl.vision_dim, wl.n_heads, wl.mlp_hidden, wl.downsample_ratio, wl.llm_dim,
                         wl.n_layers if n_layers is None else n_layers, wl.eps, wl.rope_theta,
                         A.DSV4V_F32 if wl.dtype == "f32" else A.DSV4V_BF16)


def upload_layers(inp):
    out = []
    for layer in inp.layers:
        d = {}
        for k, v in layer.items():
            d[k] = f32(v) if isinstance(v, np.ndarray) else dev(v)
        out.append(d)
    return out


def workspace(cfg, batch):
    n = A.dsv4v_workspace_size(cfg, batch)
    assert n > 0
    return torch.empty(n, dtype=torch.uint8, device="cuda")


def rel_fro(g, o):
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    return float(np.linalg.norm(g - o) / np.linalg.norm(o))


def random_bf16(shape, scale=1.0, seed=0):
    rng = np.random.default_rng(seed)
    return synth._store(rng.standard_normal(shape, dtype=np.float32) * np.float32(scale), "bf16")

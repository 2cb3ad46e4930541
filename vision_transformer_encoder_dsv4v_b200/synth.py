"""Seeded synthetic inputs for the vision-tower workloads.

This module only draws random numbers and stores them in the activation dtype; it holds none
of the tower's arithmetic.  Both the CUDA path (through the tests and the benchmark) and the
fp64 oracle consume what it returns, so the two always see bit-identical inputs.

Recipe (numpy ``default_rng(seed)``, PCG64, float32 draws):

* grids first (only the high-resolution workload draws them), then ``x``, then for every layer
  ``norm1_w, wqkv, wo, norm2_w, w_gate, w_up, w_down``, then ``final_norm_w`` (tower workloads
  only), then ``w_align`` (workloads with the aligner only);
* patch states ``x ~ N(0, 1)``; every linear weight ``~ N(0, 0.02)``; RMSNorm scales
  ``1 + N(0, 0.1)`` kept in fp32;
* bf16 workloads round activations and linear weights to bf16 with round-to-nearest-even;
  the oracle widens exactly those stored values.

Weight layouts follow ``nn.Linear``: ``[out_features, in_features]`` row-major.
``wqkv`` is ``[3D, D]`` with the q, k, v blocks stacked in that order.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass
class Workload:
    name: str
    dtype: str            # "f32" or "bf16": storage/compute dtype of activations and weights
    vision_dim: int
    n_heads: int
    mlp_hidden: int
    downsample_ratio: int
    llm_dim: int
    n_layers: int
    grids: list           # [(n_h, n_w), ...] in packing order
    seed: int
    final_norm: bool      # tower workloads apply the tower's final RMSNorm
    aligner: bool         # workloads that end with the aligner projection
    eps: float = 1e-6
    rope_theta: float = 10000.0

    @property
    def head_dim(self) -> int:
        return self.vision_dim // self.n_heads

    @property
    def n_patches(self) -> int:
        return int(sum(h * w for h, w in self.grids))

    @property
    def cu_patches(self) -> np.ndarray:
        cu = np.zeros(len(self.grids) + 1, dtype=np.int32)
        cu[1:] = np.cumsum([h * w for h, w in self.grids])
        return cu

    @property
    def n_tokens(self) -> int:
        r = self.downsample_ratio
        return int(sum(-(-h // r) * -(-w // r) for h, w in self.grids))


def _hi_res_grids(rng: np.random.Generator) -> list:
    """16 images: 15 with sides drawn uniformly from 8..64, plus one 64x64.  Redrawn until the
    packed batch holds 20 000..30 000 patches."""
    while True:
        hw = rng.integers(8, 65, size=(15, 2))
        grids = [(int(a), int(b)) for a, b in hw] + [(64, 64)]
        p = sum(a * b for a, b in grids)
        if 20000 <= p <= 30000:
            return grids


_BIG = dict(vision_dim=1024, n_heads=16, mlp_hidden=2816, downsample_ratio=2, llm_dim=4096)


def workload(idx: int) -> Workload:
    """The five workloads: 1 fp32 block + aligner (4x6); 2 bf16 block (28x28); 3 bf16 block on a
    ragged packed batch (27x37, 37x27, 10x78, 112x7); 4 bf16 32-layer tower + aligner (28x28);
    5 bf16 32-layer tower + aligner on 16 packed images (grids drawn in ``draw``)."""
    if idx == 1:
        return Workload("block+aligner fp32 4x6 D64", "f32", 64, 4, 128, 2, 128, 1,
                        [(4, 6)], 0, final_norm=False, aligner=True)
    if idx == 2:
        return Workload("block bf16 28x28", "bf16", n_layers=1, grids=[(28, 28)], seed=1,
                        final_norm=False, aligner=False, **_BIG)
    if idx == 3:
        return Workload("block bf16 packed 27x37+37x27+10x78+112x7", "bf16", n_layers=1,
                        grids=[(27, 37), (37, 27), (10, 78), (112, 7)], seed=2,
                        final_norm=False, aligner=False, **_BIG)
    if idx == 4:
        return Workload("tower32+aligner bf16 28x28", "bf16", n_layers=32, grids=[(28, 28)],
                        seed=3, final_norm=True, aligner=True, **_BIG)
    if idx == 5:
        rng = np.random.default_rng(4)
        return Workload("tower32+aligner bf16 16 images 8..64 + 64x64", "bf16", n_layers=32,
                        grids=_hi_res_grids(rng), seed=4, final_norm=True, aligner=True, **_BIG)
    raise ValueError(f"unknown workload {idx}")


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even) and return the raw bits."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    rounded = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)
    return rounded.astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits to float32 exactly."""
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Tensor:
    """One stored input: ``values`` are the exact stored numbers as float32; ``bits`` are the raw
    bf16 bits when the storage dtype is bf16 (None for fp32 storage)."""
    values: np.ndarray
    bits: np.ndarray | None = None


@dataclass
class Inputs:
    wl: Workload
    x: Tensor
    layers: list = field(default_factory=list)   # list of dict name -> Tensor
    final_norm_w: np.ndarray | None = None       # fp32 [D]
    w_align: Tensor | None = None


LAYER_KEYS = ("norm1_w", "wqkv", "wo", "norm2_w", "w_gate", "w_up", "w_down")


def _store(a32: np.ndarray, dtype: str) -> Tensor:
    if dtype == "f32":
        return Tensor(np.ascontiguousarray(a32, dtype=np.float32))
    bits = bf16_bits(a32)
    return Tensor(bf16_to_f32(bits), bits)


def draw(wl: Workload, n_layers: int | None = None) -> Inputs:
    """Draw every input of ``wl`` in the documented order.  ``n_layers`` < wl.n_layers draws only
    the first layers (the stream is consumed in layer order, so those layers are identical to the
    full draw's); the final norm and aligner weights are then not drawn."""
    rng = np.random.default_rng(wl.seed)
    if wl.name.startswith("tower32+aligner bf16 16 images"):
        _hi_res_grids(rng)  # consume the grid draw so x follows it in the stream
    D, F = wl.vision_dim, wl.mlp_hidden
    P = wl.n_patches
    n = wl.n_layers if n_layers is None else n_layers
    inp = Inputs(wl, _store(rng.standard_normal((P, D), dtype=np.float32), wl.dtype))
    lin = lambda o, i: _store(rng.standard_normal((o, i), dtype=np.float32) * np.float32(0.02), wl.dtype)
    scale = lambda: (np.float32(1.0) + rng.standard_normal(D, dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    for _ in range(n):
        layer = {}
        layer["norm1_w"] = scale()
        layer["wqkv"] = lin(3 * D, D)
        layer["wo"] = lin(D, D)
        layer["norm2_w"] = scale()
        layer["w_gate"] = lin(F, D)
        layer["w_up"] = lin(F, D)
        layer["w_down"] = lin(D, F)
        inp.layers.append(layer)
    if n == wl.n_layers:
        if wl.final_norm:
            inp.final_norm_w = scale()
        if wl.aligner:
            r = wl.downsample_ratio
            inp.w_align = lin(wl.llm_dim, r * r * D)
    return inp


def algorithmic_flops(wl: Workload, n_layers: int | None = None, aligner: bool | None = None) -> float:
    """Counted work: per block sum_i N_i (8 D^2 + 6 D F) + 4 N_i^2 D; aligner 2 T r^2 D E."""
    D, F = wl.vision_dim, wl.mlp_hidden
    L = wl.n_layers if n_layers is None else n_layers
    per_block = sum(h * w * (8 * D * D + 6 * D * F) + 4 * (h * w) ** 2 * D for h, w in wl.grids)
    total = float(L) * per_block
    if wl.aligner if aligner is None else aligner:
        r = wl.downsample_ratio
        total += 2.0 * wl.n_tokens * r * r * D * wl.llm_dim
    return total


def place_spans(layouts, n_seqs: int, seq_len: int, seed: int, max_gap: int = 40, pad_every: int = 0,
                balance: bool = False) -> np.ndarray:
    """A seeded [n_seqs, seq_len] int32 pseudo-token type array: the given per-image layouts
    (int32 arrays, in image order) placed left to right into text (-1) sequences, each preceded
    by a text gap drawn uniformly from 0..max_gap.  By default an image moves to the next
    sequence when it does not fit; with balance=True image i goes to sequence
    floor(i * n_seqs / n_images), so the sequences hold contiguous, near-equal groups.  With
    pad_every = k > 0, every k-th image gets one type-4 entry inserted before its last entry (a
    filler inside the span).  Raises ValueError if the images do not fit."""
    rng = np.random.default_rng(seed)
    out = np.full((n_seqs, seq_len), -1, dtype=np.int32)
    s, pos = 0, 0
    n_img = len(layouts)
    for i, lay in enumerate(layouts):
        lay = np.asarray(lay, dtype=np.int32)
        if pad_every and i % pad_every == pad_every - 1:
            lay = np.concatenate([lay[:-1], np.array([4], np.int32), lay[-1:]])
        gap = int(rng.integers(0, max_gap + 1))
        target = i * n_seqs // n_img if balance else s
        if target != s:
            s, pos = target, 0
        elif not balance and pos + gap + len(lay) > seq_len:
            s, pos = s + 1, 0
        if s >= n_seqs or pos + gap + len(lay) > seq_len:
            raise ValueError(f"image {i} ({len(lay)} positions) does not fit")
        out[s, pos + gap: pos + gap + len(lay)] = lay
        pos += gap + len(lay)
    return out

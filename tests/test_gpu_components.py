"""Parity of each kernel of the path with the fp64 oracle, called through the C ABI.

Tolerances: a GEMM-shaped step (fp32 accumulation, epilogue in fp32, one rounding to bf16) must
satisfy |gpu - oracle| <= 2^-8 |oracle| + abs_floor element by element (one bf16 rounding is at
most 2^-9 relative); attention rounds P to bf16 before the PV product, so it is held to a
relative Frobenius error of 1e-2 plus an element-wise bound."""
import numpy as np
import pytest
import torch

from gpu_util import config_of, dev, f32, random_bf16, rel_fro, to_np, workspace
from oracle import dsv4v_oracle as O
from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
from vision_transformer_encoder_dsv4v_b200 import synth

pytestmark = pytest.mark.gpu

BIG = dict(vision_dim=1024, n_heads=16, mlp_hidden=2816, downsample_ratio=2, llm_dim=4096, n_layers=1)
GRID_SETS = {
    "28x28": [(28, 28)],
    "ragged4": [(27, 37), (37, 27), (10, 78), (112, 7)],
    "tiny": [(1, 1)],
    "lines": [(1, 37), (37, 1), (3, 5)],
    "mixed": [(3, 5), (1, 1), (64, 64), (9, 14)],
    # last key tile holding 40, 70, 96, 97, 33 and 64 keys: every 32-key chunk boundary
    "chunks": [(5, 8), (7, 10), (12, 8), (1, 97), (3, 11), (16, 12)],
}


def cfg_bf16(**kw):
    d = dict(BIG)
    d.update(kw)
    return A.make_config(d["vision_dim"], d["n_heads"], d["mlp_hidden"], d["downsample_ratio"], d["llm_dim"],
                         d["n_layers"], 1e-6, 10000.0, A.DSV4V_BF16)


def assert_bf16_close(g, o, abs_floor=1e-5, rel=2.0 ** -8):
    g = np.asarray(g, dtype=np.float64)
    o = np.asarray(o, dtype=np.float64)
    bad = np.abs(g - o) > rel * np.abs(o) + abs_floor
    assert not bad.any(), f"{bad.sum()} of {bad.size} elements outside bf16 rounding; max err {np.abs(g - o).max()}"


@pytest.mark.parametrize("name", list(GRID_SETS))
def test_rope2d_table(name):
    grids = GRID_SETS[name]
    b = A.BatchRef(grids)
    cos = torch.empty(b.n_patches, 32, device="cuda")
    sin = torch.empty_like(cos)
    A.dsv4v_rope2d_table(cfg_bf16(), b, cos, sin)
    c_o, s_o = O.packed_cos_sin(grids, 32, 10000.0)
    assert np.abs(to_np(cos) - c_o).max() < 5e-5
    assert np.abs(to_np(sin) - s_o).max() < 5e-5


@pytest.mark.parametrize("rows", [1, 777, 4097])
def test_rmsnorm_bf16(rows):
    x = random_bf16((rows, 1024), 3.0, seed=rows)
    w = (1 + 0.1 * np.random.default_rng(rows).standard_normal(1024)).astype(np.float32)
    y = torch.empty(rows, 1024, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_rmsnorm(cfg_bf16(), rows, dev(x), f32(w), y)
    assert_bf16_close(to_np(y), O.rmsnorm(x.values, w, 1e-6), abs_floor=1e-6)


def test_rmsnorm_f32_in_place():
    cfg = A.make_config(64, 4, 128, 2, 128, 1, 1e-6, 10000.0, A.DSV4V_F32)
    x = np.random.default_rng(5).standard_normal((50, 64)).astype(np.float32)
    w = (1 + 0.1 * np.random.default_rng(6).standard_normal(64)).astype(np.float32)
    xt = f32(x)
    A.dsv4v_rmsnorm(cfg, 50, xt, f32(w), xt)
    assert np.abs(to_np(xt) - O.rmsnorm(x, w, 1e-6)).max() < 1e-5


@pytest.mark.parametrize("name", ["28x28", "ragged4", "tiny", "lines"])
def test_qkv_rope(name):
    grids = GRID_SETS[name]
    b = A.BatchRef(grids)
    cfg = cfg_bf16()
    P = b.n_patches
    y = random_bf16((P, 1024), 1.0, seed=11)
    wqkv = random_bf16((3072, 1024), 0.02, seed=12)
    c_o, s_o = O.packed_cos_sin(grids, 32, 10000.0)
    qkv = torch.empty(P, 3072, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_qkv_rope(cfg, b, dev(y), dev(wqkv), f32(c_o), f32(s_o), qkv, workspace(cfg, b))
    q, k, v = O.qkv_rope(y.values, wqkv.values, c_o.astype(np.float32), s_o.astype(np.float32), 16)
    want = np.concatenate([q.reshape(P, -1), k.reshape(P, -1), v.reshape(P, -1)], axis=1)
    assert_bf16_close(to_np(qkv), want, abs_floor=2e-5)


@pytest.mark.parametrize("name,scale", [("28x28", 1.0), ("ragged4", 1.0), ("mixed", 1.0), ("lines", 1.0),
                                        ("tiny", 1.0), ("chunks", 1.0), ("28x28", 3.0)])
def test_attention(name, scale):
    grids = GRID_SETS[name]
    b = A.BatchRef(grids)
    P = b.n_patches
    qkv = random_bf16((P, 3072), scale, seed=21)
    out = torch.empty(P, 1024, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_attention(cfg_bf16(), b, dev(qkv), out)
    qv = qkv.values.reshape(P, 3, 16, 64)
    want = O.attention_packed(qv[:, 0], qv[:, 1], qv[:, 2], grids)
    got = to_np(out)
    assert rel_fro(got, want) < 1e-2
    assert np.abs(got - want).max() < 2e-2 * max(1.0, np.abs(want).max())


@pytest.mark.parametrize("rows,k", [(784, 1024), (784, 2816), (3562, 1024), (1, 2816), (129, 1024)])
def test_linear_residual(rows, k):
    cfg = cfg_bf16()
    a = random_bf16((rows, k), 1.0, seed=31)
    w = random_bf16((1024, k), 0.02, seed=32)
    x = random_bf16((rows, 1024), 1.0, seed=33)
    xt = dev(x)
    ws = torch.empty(A.dsv4v_workspace_size(cfg, A.BatchRef([(rows, 1)])), dtype=torch.uint8, device="cuda")
    A.dsv4v_linear_residual(cfg, rows, k, dev(a), dev(w), xt, ws)
    want = x.values.astype(np.float64) + a.values.astype(np.float64) @ w.values.astype(np.float64).T
    assert_bf16_close(to_np(xt), want, abs_floor=2e-5)


# 784, 1000 (ragged last row tile) and 1152 rows take 176-column tiles, one per CTA
@pytest.mark.parametrize("rows", [784, 1000, 1152, 3562, 1, 200])
def test_swiglu(rows):
    cfg = cfg_bf16()
    y = random_bf16((rows, 1024), 1.0, seed=41)
    wg = random_bf16((2816, 1024), 0.02, seed=42)
    wu = random_bf16((2816, 1024), 0.02, seed=43)
    h = torch.empty(rows, 2816, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.dsv4v_workspace_size(cfg, A.BatchRef([(rows, 1)])), dtype=torch.uint8, device="cuda")
    A.dsv4v_swiglu(cfg, rows, dev(y), dev(wg), dev(wu), h, ws)
    yy = y.values.astype(np.float64)
    want = O.silu(yy @ wg.values.astype(np.float64).T) * (yy @ wu.values.astype(np.float64).T)
    assert_bf16_close(to_np(h), want, abs_floor=2e-5)


@pytest.mark.parametrize("grids", [[(28, 28)], [(27, 37), (37, 27), (10, 78), (112, 7)], [(3, 5), (1, 1), (4, 6)]])
def test_aligner_bf16(grids):
    cfg = cfg_bf16()
    b = A.BatchRef(grids)
    P = b.n_patches
    x = random_bf16((P, 1024), 1.0, seed=51)
    wa = random_bf16((4096, 4096), 0.02, seed=52)
    T = A.dsv4v_aligner_tokens(cfg, b)
    out = torch.empty(T, 4096, dtype=torch.bfloat16, device="cuda")
    cu_tok = torch.zeros(len(grids) + 1, dtype=torch.int32)
    A.dsv4v_aligner_forward(cfg, b, dev(x), dev(wa), out, workspace(cfg, b), cu_tokens_host=cu_tok)
    want, cu_o = O.aligner_forward(x.values, wa.values, grids, 2)
    assert list(cu_tok.numpy()) == list(cu_o)
    assert_bf16_close(to_np(out), want, abs_floor=2e-5)


# Shapes large enough that the planner runs the block GEMMs on CTA pairs (256-row tiles split
# between two SMs, tcgen05 cta_group::2).  The oracle is evaluated on sampled rows: both CTAs'
# halves of several pair tiles, the pair-tile boundaries and the ragged tail.
def _pair_rows(m, seed):
    rng = np.random.default_rng(seed)
    edges = [0, 1, 127, 128, 129, 255, 256, 257, 383, 384, 511, 512]
    tail = [m - 1 - i for i in range(0, 260, 37)] + [(m // 256) * 256 - 1, (m // 256) * 256]
    picks = rng.choice(m, size=64, replace=False).tolist()
    return np.array(sorted({r for r in edges + tail + picks if 0 <= r < m}))


@pytest.mark.parametrize("k", [1024, 2816])
def test_linear_residual_pair_tiles(k):
    rows = 25985
    cfg = cfg_bf16()
    a = random_bf16((rows, k), 1.0, seed=61)
    w = random_bf16((1024, k), 0.02, seed=62)
    x = random_bf16((rows, 1024), 1.0, seed=63)
    xt = dev(x)
    ws = torch.empty(A.dsv4v_workspace_size(cfg, A.BatchRef([(rows, 1)])), dtype=torch.uint8, device="cuda")
    A.dsv4v_linear_residual(cfg, rows, k, dev(a), dev(w), xt, ws)
    assert A.dsv4v_device_error() == 0
    r = _pair_rows(rows, 64)
    want = x.values[r].astype(np.float64) + a.values[r].astype(np.float64) @ w.values.astype(np.float64).T
    assert_bf16_close(to_np(xt)[r], want, abs_floor=2e-5)


def test_swiglu_pair_tiles():
    rows = 9001
    cfg = cfg_bf16()
    y = random_bf16((rows, 1024), 1.0, seed=71)
    wg = random_bf16((2816, 1024), 0.02, seed=72)
    wu = random_bf16((2816, 1024), 0.02, seed=73)
    h = torch.empty(rows, 2816, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.dsv4v_workspace_size(cfg, A.BatchRef([(rows, 1)])), dtype=torch.uint8, device="cuda")
    A.dsv4v_swiglu(cfg, rows, dev(y), dev(wg), dev(wu), h, ws)
    assert A.dsv4v_device_error() == 0
    r = _pair_rows(rows, 74)
    yy = y.values[r].astype(np.float64)
    want = O.silu(yy @ wg.values.astype(np.float64).T) * (yy @ wu.values.astype(np.float64).T)
    assert_bf16_close(to_np(h)[r], want, abs_floor=2e-5)


def test_qkv_rope_pair_tiles():
    grids = [(64, 64), (64, 64), (30, 31)]
    b = A.BatchRef(grids)
    cfg = cfg_bf16()
    P = b.n_patches
    y = random_bf16((P, 1024), 1.0, seed=81)
    wqkv = random_bf16((3072, 1024), 0.02, seed=82)
    c_o, s_o = O.packed_cos_sin(grids, 32, 10000.0)
    qkv = torch.empty(P, 3072, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_qkv_rope(cfg, b, dev(y), dev(wqkv), f32(c_o), f32(s_o), qkv, workspace(cfg, b))
    assert A.dsv4v_device_error() == 0
    r = _pair_rows(P, 84)
    q, k, v = O.qkv_rope(y.values[r], wqkv.values, c_o[r].astype(np.float32), s_o[r].astype(np.float32), 16)
    want = np.concatenate([q.reshape(len(r), -1), k.reshape(len(r), -1), v.reshape(len(r), -1)], axis=1)
    assert_bf16_close(to_np(qkv)[r], want, abs_floor=2e-5)


# Patch embedding (next step before the tower): flattened (3, p, p) patches through `proj`.
@pytest.mark.parametrize("rows,patch,bias,ld", [(784, 16, True, 0), (784, 14, False, 592), (1, 14, True, 592),
                                                (3562, 16, False, 0), (130, 14, True, 600)])
def test_patch_embed_bf16(rows, patch, bias, ld):
    cfg = cfg_bf16()
    k = 3 * patch * patch
    width = ld if ld else k
    pix = random_bf16((rows, width), 1.0, seed=91)
    w = random_bf16((1024, width), 0.02, seed=92)
    if width > k:  # the padding past K must never be read: make it loud
        for t in (pix, w):
            t.bits[:, k:] = synth.bf16_bits(np.full((t.bits.shape[0], width - k), 1.0e4, dtype=np.float32))
            t.values[:, k:] = 1.0e4
    b = np.random.default_rng(93).normal(size=1024).astype(np.float32) if bias else None
    out = torch.empty(rows, 1024, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_patch_embed(cfg, rows, patch, patch, dev(pix), dev(w), f32(b) if bias else None, out, ld, ld)
    assert A.dsv4v_device_error() == 0
    want = O.patch_embed(pix.values[:, :k].reshape(rows, 3, patch, patch), w.values[:, :k], b)
    assert_bf16_close(to_np(out), want, abs_floor=2e-5)


def test_patch_embed_f32():
    cfg = A.make_config(64, 4, 128, 2, 128, 1, 1e-6, 10000.0, A.DSV4V_F32)
    rows, patch = 24, 4
    rng = np.random.default_rng(94)
    pix = rng.normal(size=(rows, 3, patch, patch)).astype(np.float32)
    w = (0.1 * rng.normal(size=(64, 3 * patch * patch))).astype(np.float32)
    b = rng.normal(size=64).astype(np.float32)
    out = torch.empty(rows, 64, dtype=torch.float32, device="cuda")
    A.dsv4v_patch_embed(cfg, rows, patch, patch, f32(pix.reshape(rows, -1)), f32(w), f32(b), out)
    want = O.patch_embed(pix, w, b)
    assert np.abs(out.cpu().numpy().astype(np.float64) - want).max() < 1e-4


# PatchMerger projector (the second aligner on the pages): LayerNorm per patch, r x r merge,
# Linear + GELU, Linear.  Two GEMMs with a bf16 intermediate: relative Frobenius error <= 1e-2
# plus an element-wise bound.
@pytest.mark.parametrize("grids", [[(28, 28)], [(3, 5), (1, 1), (4, 6)], [(27, 37), (37, 27), (10, 78), (112, 7)]])
def test_patch_merger_bf16(grids):
    cfg = cfg_bf16()
    b = A.BatchRef(grids)
    P = b.n_patches
    rng = np.random.default_rng(55)
    x = random_bf16((P, 1024), 1.0, seed=56)
    ln_w = (1 + 0.1 * rng.normal(size=1024)).astype(np.float32)
    ln_b = (0.1 * rng.normal(size=1024)).astype(np.float32)
    w1 = random_bf16((4096, 4096), 0.02, seed=57)
    b1 = (0.1 * rng.normal(size=4096)).astype(np.float32)
    w2 = random_bf16((4096, 4096), 0.02, seed=58)
    b2 = (0.1 * rng.normal(size=4096)).astype(np.float32)
    T = A.dsv4v_aligner_tokens(cfg, b)
    out = torch.empty(T, 4096, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(A.dsv4v_patch_merger_workspace_size(cfg, b), dtype=torch.uint8, device="cuda")
    A.dsv4v_patch_merger_forward(cfg, b, dev(x), f32(ln_w), f32(ln_b), dev(w1), f32(b1), dev(w2), f32(b2), out, ws)
    assert A.dsv4v_device_error() == 0
    want, _ = O.patch_merger(x.values, grids, 2, ln_w, ln_b, w1.values, b1, w2.values, b2, eps=1e-6)
    got = to_np(out)
    assert rel_fro(got, want) < 1e-2
    assert np.abs(got - want).max() < 3e-2 * max(1.0, np.abs(want).max())


def test_patch_merger_f32():
    cfg = A.make_config(64, 4, 128, 2, 128, 1, 1e-6, 10000.0, A.DSV4V_F32)
    grids = [(4, 6), (3, 5)]
    b = A.BatchRef(grids)
    P = b.n_patches
    rng = np.random.default_rng(59)
    x = rng.normal(size=(P, 64)).astype(np.float32)
    ln_w = (1 + 0.1 * rng.normal(size=64)).astype(np.float32)
    ln_b = (0.1 * rng.normal(size=64)).astype(np.float32)
    w1 = (0.05 * rng.normal(size=(256, 256))).astype(np.float32)
    b1 = (0.1 * rng.normal(size=256)).astype(np.float32)
    w2 = (0.05 * rng.normal(size=(128, 256))).astype(np.float32)
    b2 = (0.1 * rng.normal(size=128)).astype(np.float32)
    T = A.dsv4v_aligner_tokens(cfg, b)
    out = torch.empty(T, 128, dtype=torch.float32, device="cuda")
    ws = torch.empty(A.dsv4v_patch_merger_workspace_size(cfg, b), dtype=torch.uint8, device="cuda")
    A.dsv4v_patch_merger_forward(cfg, b, f32(x), f32(ln_w), f32(ln_b), f32(w1), f32(b1), f32(w2), f32(b2), out, ws)
    want, _ = O.patch_merger(x, grids, 2, ln_w, ln_b, w1, b1, w2, b2, eps=1e-6)
    assert np.abs(out.cpu().numpy().astype(np.float64) - want).max() < 1e-4

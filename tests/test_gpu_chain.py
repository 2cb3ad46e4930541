"""The two launch sequences of the bf16 blocks -- one kernel per GEMM, and the persistent chain
kernel that runs the output projection, SwiGLU, the down projection and the next block's q|k|v
projection in one launch -- each against the fp64 oracle, and against each other.

Both compute the same block with the same roundings; they may split the GEMMs' K dimension
differently, so fp32 sums can be added in another order and a few bf16 results can differ by a
rounding step.  The bars are the oracle tolerances (1e-2 per block, 3e-2 over a tower)."""
import numpy as np
import pytest
import torch

from gpu_util import config_of, dev, f32, rel_fro, to_np, upload_layers, workspace
from oracle import dsv4v_oracle as O
from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
from vision_transformer_encoder_dsv4v_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def restore_path():
    yield
    A.dsv4v_set_tower_path(A.PATH_AUTO)


def _block(inp, path):
    A.dsv4v_set_tower_path(path)
    wl = inp.wl
    cfg = config_of(wl, n_layers=1)
    b = A.BatchRef(wl.grids)
    assert A.dsv4v_tower_path(cfg, b) == path
    cos = torch.empty(b.n_patches, wl.head_dim // 2, device="cuda")
    sin = torch.empty_like(cos)
    A.dsv4v_rope2d_table(cfg, b, cos, sin)
    x = dev(inp.x)
    layer = upload_layers(inp)[0]
    A.dsv4v_block_forward(cfg, b, A.block_weights(layer), cos, sin, x, workspace(cfg, b))
    assert A.dsv4v_device_error() == 0
    return to_np(x)


def _oracle_block(inp):
    wl = inp.wl
    cos, sin = O.packed_cos_sin(wl.grids, wl.head_dim // 2, wl.rope_theta)
    layer = {k: (v.values if hasattr(v, "values") else v) for k, v in inp.layers[0].items()}
    return O.block_forward(inp.x.values, layer, cos, sin, wl.grids, wl.n_heads, wl.eps)


@pytest.mark.parametrize("grids", [[(28, 28)], [(27, 37), (37, 27), (10, 78), (112, 7)], [(1, 1)],
                                   [(1, 1), (3, 5), (9, 14)], [(2, 64), (64, 2)], [(8, 8)] * 40 + [(5, 3)] * 25])
def test_chain_block_matches_oracle_and_kernel_path(grids):
    wl = synth.Workload("chain", "bf16", 1024, 16, 2816, 2, 4096, 1, grids, 21, False, False)
    inp = synth.draw(wl)
    want = _oracle_block(inp)
    got_chain = _block(inp, A.PATH_CHAIN)
    got_kern = _block(inp, A.PATH_KERNELS)
    e_c, e_k = rel_fro(got_chain, want), rel_fro(got_kern, want)
    d_c = rel_fro(got_chain - inp.x.values, want - inp.x.values)
    print(f"{grids[:4]}: chain {e_c:.3e} (delta {d_c:.3e}), kernels {e_k:.3e}, "
          f"chain vs kernels {rel_fro(got_chain, got_kern):.3e}")
    assert e_c <= 1e-2 and d_c <= 3e-2
    assert e_k <= 1e-2
    # the two sequences round the same products: they agree far more closely than either bar
    assert rel_fro(got_chain, got_kern) <= 2e-3
    # the chain path is deterministic (split partials are added in split order)
    assert np.array_equal(got_chain, _block(inp, A.PATH_CHAIN))


def test_chain_tower_three_layers_matches_oracle_and_kernel_path():
    wl = synth.workload(4)
    inp = synth.draw(wl, n_layers=3)
    cfg = config_of(wl, n_layers=3)
    b = A.BatchRef(wl.grids)
    layers = upload_layers(inp)
    keep = [A.block_weights(l) for l in layers]
    fnw = f32(1.0 + 0.1 * np.random.default_rng(5).standard_normal(wl.vision_dim))
    outs = {}
    for path in (A.PATH_CHAIN, A.PATH_KERNELS):
        A.dsv4v_set_tower_path(path)
        x = dev(inp.x)
        A.dsv4v_tower_forward(cfg, b, keep, fnw, x, workspace(cfg, b))
        assert A.dsv4v_device_error() == 0
        outs[path] = to_np(x)
    lay = [{k: (v.values if hasattr(v, "values") else v) for k, v in l.items()} for l in inp.layers]
    want = O.tower_forward(inp.x.values, lay, fnw.cpu().numpy(), wl.grids, wl.n_heads, wl.rope_theta, wl.eps)
    e_c, e_k = rel_fro(outs[A.PATH_CHAIN], want), rel_fro(outs[A.PATH_KERNELS], want)
    print(f"3-layer tower: chain {e_c:.3e}, kernels {e_k:.3e}")
    assert e_c <= 3e-2 and e_k <= 3e-2
    assert rel_fro(outs[A.PATH_CHAIN], outs[A.PATH_KERNELS]) <= 5e-3


def test_chain_profiled_tower_records_attention_and_chain():
    A.dsv4v_set_tower_path(A.PATH_CHAIN)
    wl = synth.workload(4)
    inp = synth.draw(wl, n_layers=2)
    cfg = config_of(wl, n_layers=2)
    b = A.BatchRef(wl.grids)
    ws = workspace(cfg, b)
    layers = upload_layers(inp)
    keep = [A.block_weights(l) for l in layers]
    x1, x2 = dev(inp.x), dev(inp.x)
    A.dsv4v_tower_forward(cfg, b, keep, None, x1, ws)
    kinds = A.PROFILE_KINDS
    events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * len(kinds) * 2)]
    for e in events:
        e.record()
    torch.cuda.synchronize()
    A.dsv4v_tower_forward_profiled(cfg, b, keep, None, x2, ws, events)
    torch.cuda.synchronize()
    assert torch.equal(x1, x2)
    for l in range(2):
        for k in ("attention", "chain"):
            i = (l * len(kinds) + kinds.index(k)) * 2
            assert events[i].elapsed_time(events[i + 1]) > 0.0

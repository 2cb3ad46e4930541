"""Whole-path parity with the fp64 oracle on the five seeded workloads, plus the structural
properties of packing (isolation, permutation, determinism) and the boundary's error paths.

Bars: the fp32 workload within 1e-4 max abs; a bf16 block within 1e-2 relative Frobenius error;
the bf16 32-layer tower and the aligner within 3e-2."""
import numpy as np
import pytest
import torch

from gpu_util import config_of, dev, f32, random_bf16, rel_fro, to_np, upload_layers, workspace
from oracle import dsv4v_oracle as O
from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
from vision_transformer_encoder_dsv4v_b200 import synth

pytestmark = pytest.mark.gpu


def run_block(inp, x_override=None, grids=None):
    wl = inp.wl
    grids = wl.grids if grids is None else grids
    cfg = config_of(wl, n_layers=1)
    b = A.BatchRef(grids)
    hd2 = wl.head_dim // 2
    cos = torch.empty(b.n_patches, hd2, device="cuda")
    sin = torch.empty_like(cos)
    A.dsv4v_rope2d_table(cfg, b, cos, sin)
    x = dev(inp.x) if x_override is None else x_override
    layer = upload_layers(inp)[0]
    A.dsv4v_block_forward(cfg, b, A.block_weights(layer), cos, sin, x, workspace(cfg, b))
    assert A.dsv4v_device_error() == 0
    return x


def oracle_block(inp, x=None, grids=None):
    wl = inp.wl
    grids = wl.grids if grids is None else grids
    cos, sin = O.packed_cos_sin(grids, wl.head_dim // 2, wl.rope_theta)
    layer = {k: (v.values if hasattr(v, "values") else v) for k, v in inp.layers[0].items()}
    return O.block_forward(inp.x.values if x is None else x, layer, cos, sin, grids, wl.n_heads, wl.eps)


# ------------------------------------------------------------------------------ workload 1 (fp32)
def test_workload1_fp32_block_and_aligner():
    wl = synth.workload(1)
    inp = synth.draw(wl)
    x = run_block(inp)
    want = oracle_block(inp)
    assert np.abs(to_np(x) - want).max() <= 1e-4
    cfg = config_of(wl)
    b = A.BatchRef(wl.grids)
    out = torch.empty(wl.n_tokens, wl.llm_dim, device="cuda")
    A.dsv4v_aligner_forward(cfg, b, x, dev(inp.w_align), out, workspace(cfg, b))
    want_a, _ = O.aligner_forward(want, inp.w_align.values, wl.grids, wl.downsample_ratio)
    assert np.abs(to_np(out) - want_a).max() <= 1e-4
    # the tower entry point with one layer and no final norm is the same block
    x2 = dev(inp.x)
    layer = upload_layers(inp)[0]  # keep the device tensors alive across the call
    A.dsv4v_tower_forward(cfg, b, [A.block_weights(layer)], None, x2, workspace(cfg, b))
    assert np.abs(to_np(x2) - want).max() <= 1e-4


# ------------------------------------------------------------------------------ workloads 2, 3
@pytest.mark.parametrize("idx", [2, 3])
def test_bf16_block_workloads(idx):
    wl = synth.workload(idx)
    inp = synth.draw(wl)
    got = to_np(run_block(inp))
    want = oracle_block(inp)
    err = rel_fro(got, want)
    delta_err = rel_fro(got - inp.x.values, want - inp.x.values)
    print(f"workload {idx}: rel fro {err:.3e}, block-delta rel fro {delta_err:.3e}")
    assert err <= 1e-2
    assert delta_err <= 3e-2


@pytest.mark.parametrize("grids", [[(1, 1)], [(1, 37)], [(37, 1)], [(3, 5), (1, 1), (64, 64), (9, 14)],
                                   [(8, 8)] * 40 + [(5, 3)] * 25])
def test_bf16_block_edge_grids(grids):
    wl = synth.Workload("edge", "bf16", 1024, 16, 2816, 2, 4096, 1, grids, 7, False, False)
    inp = synth.draw(wl)
    got = to_np(run_block(inp))
    want = oracle_block(inp)
    assert rel_fro(got, want) <= 1e-2
    assert rel_fro(got - inp.x.values, want - inp.x.values) <= 3e-2


def test_packing_isolation_permutation_determinism():
    wl = synth.workload(3)
    inp = synth.draw(wl)
    cu = wl.cu_patches
    base = to_np(run_block(inp))
    again = to_np(run_block(inp))
    assert np.array_equal(base, again), "two identical calls differ"
    # change image 2's patches: images 0, 1, 3 keep bitwise identical outputs
    x_mod = dev(inp.x)
    x_mod[cu[2]:cu[3]] = torch.randn(cu[3] - cu[2], 1024, device="cuda").to(torch.bfloat16)
    mod = to_np(run_block(inp, x_override=x_mod))
    for i in (0, 1, 3):
        assert np.array_equal(mod[cu[i]:cu[i + 1]], base[cu[i]:cu[i + 1]]), f"image {i} changed"
    assert not np.array_equal(mod[cu[2]:cu[3]], base[cu[2]:cu[3]])
    # permute the images: outputs permute with them
    order = [3, 1, 0, 2]
    grids_p = [wl.grids[i] for i in order]
    xs = dev(inp.x)
    x_perm = torch.cat([xs[cu[i]:cu[i + 1]] for i in order])
    perm = to_np(run_block(inp, x_override=x_perm, grids=grids_p))
    want_perm = np.concatenate([base[cu[i]:cu[i + 1]] for i in order])
    assert np.abs(perm - want_perm).max() <= 2.0 ** -7 * np.abs(want_perm).max()
    # each image alone agrees with its slice of the packed run
    for i in range(4):
        alone = to_np(run_block(inp, x_override=xs[cu[i]:cu[i + 1]].clone(), grids=[wl.grids[i]]))
        assert rel_fro(alone, base[cu[i]:cu[i + 1]]) < 5e-3


# ------------------------------------------------------------------------------ workload 4
@pytest.fixture(scope="module")
def workload4():
    wl = synth.workload(4)
    inp = synth.draw(wl)
    tower_o, align_o = O.encode(inp)
    return wl, inp, tower_o, align_o


def run_tower_and_aligner(wl, inp):
    cfg = config_of(wl)
    b = A.BatchRef(wl.grids)
    ws = workspace(cfg, b)
    layers = upload_layers(inp)
    keep = [A.block_weights(l) for l in layers]
    x = dev(inp.x)
    A.dsv4v_tower_forward(cfg, b, keep, f32(inp.final_norm_w), x, ws)
    out = torch.empty(A.dsv4v_aligner_tokens(cfg, b), wl.llm_dim, dtype=torch.bfloat16, device="cuda")
    A.dsv4v_aligner_forward(cfg, b, x, dev(inp.w_align), out, ws)
    assert A.dsv4v_device_error() == 0
    return to_np(x), to_np(out)


@pytest.mark.parametrize("path", [A.PATH_KERNELS, A.PATH_CHAIN])
def test_profiled_tower_matches_plain(path):
    """dsv4v_tower_forward_profiled computes the same tower (bitwise) and records the events of
    the kernel classes of the launch sequence in use."""
    A.dsv4v_set_tower_path(path)
    try:
        wl = synth.workload(4)
        inp = synth.draw(wl, n_layers=3)
        cfg = config_of(wl, n_layers=3)
        b = A.BatchRef(wl.grids)
        ws = workspace(cfg, b)
        layers = upload_layers(inp)
        keep = [A.block_weights(l) for l in layers]
        x1, x2 = dev(inp.x), dev(inp.x)
        A.dsv4v_tower_forward(cfg, b, keep, None, x1, ws)
        kinds = A.PROFILE_KINDS
        events = [torch.cuda.Event(enable_timing=True) for _ in range(3 * len(kinds) * 2)]
        for e in events:
            e.record()
        torch.cuda.synchronize()
        A.dsv4v_tower_forward_profiled(cfg, b, keep, None, x2, ws, events)
        torch.cuda.synchronize()
        assert torch.equal(x1, x2)
        active = ("attention", "chain") if path == A.PATH_CHAIN else ("qkv", "attention", "out", "swiglu", "down")
        for l in range(3):
            for k in active:
                i = (l * len(kinds) + kinds.index(k)) * 2
                assert events[i].elapsed_time(events[i + 1]) > 0.0
    finally:
        A.dsv4v_set_tower_path(A.PATH_AUTO)


def test_graph_replay_matches_direct():
    """Repeated step calls with identical arguments on a side stream replay a CUDA graph (the
    first call launches directly, the second captures and replays, later calls replay).  Every
    call's tower and aligner output equals the direct launches' bitwise, also when the input
    behind the same pointer alternates between two values (the graph reads it when it runs)."""
    wl = synth.workload(4)
    inp = synth.draw(wl, n_layers=3)
    cfg = config_of(wl, n_layers=3)
    b = A.BatchRef(wl.grids)
    ws = workspace(cfg, b)
    layers = upload_layers(inp)
    keep = [A.block_weights(l) for l in layers]
    r, D = wl.downsample_ratio, wl.vision_dim
    fnw = f32(np.linspace(0.5, 1.5, D))
    wa = dev(random_bf16((wl.llm_dim, r * r * D), 0.02, seed=5))
    xs = [dev(inp.x), (dev(inp.x).float() * -0.5).to(torch.bfloat16)]
    xbuf = torch.empty_like(xs[0])
    out = torch.empty(A.dsv4v_aligner_tokens(cfg, b), wl.llm_dim, dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()

    def step(i):
        with torch.cuda.stream(s):
            xbuf.copy_(xs[i % 2])
        A.dsv4v_tower_forward(cfg, b, keep, fnw, xbuf, ws, stream=s.cuda_stream)
        A.dsv4v_aligner_forward(cfg, b, xbuf, wa, out, ws, stream=s.cuda_stream)
        s.synchronize()
        assert A.dsv4v_device_error() == 0
        return xbuf.clone(), out.clone()

    try:
        A.dsv4v_release_graphs()
        A.dsv4v_set_graph_replay(False)
        ref = [step(0), step(1)]
        A.dsv4v_set_graph_replay(True)
        for i in range(6):
            got = step(i)
            assert torch.equal(got[0], ref[i % 2][0]) and torch.equal(got[1], ref[i % 2][1]), i
        assert not torch.equal(ref[0][1], ref[1][1])
    finally:
        A.dsv4v_set_graph_replay(True)
        A.dsv4v_release_graphs()


def test_workload4_tower_aligner(workload4):
    wl, inp, tower_o, align_o = workload4
    tower_g, align_g = run_tower_and_aligner(wl, inp)
    e_t, e_a = rel_fro(tower_g, tower_o), rel_fro(align_g, align_o)
    print(f"workload 4: tower rel fro {e_t:.3e}, aligner rel fro {e_a:.3e}")
    assert e_t <= 3e-2 and e_a <= 3e-2


# ------------------------------------------------------------------------------ workload 5
def test_workload5_images_against_oracle():
    """Full 16-image batch on the GPU in the benchmark's launch configuration.  Images never
    interact, so each image's rows of the packed result are exactly what the oracle computes for
    that image alone; the oracle runs, alone, on the three smallest images, the two closest to
    1000 patches (the size class of the pages' validation grids), the largest odd (zero-padded)
    grid and the 64x64 image (4096 patches: 32 key tiles, paired query tiles)."""
    wl = synth.workload(5)
    inp = synth.draw(wl)
    tower_g, align_g = run_tower_and_aligner(wl, inp)
    cu = wl.cu_patches
    r = wl.downsample_ratio
    tok = np.cumsum([0] + [-(-h // r) * -(-w // r) for h, w in wl.grids])
    sizes = [h * w for h, w in wl.grids]
    by_size = sorted(range(len(sizes)), key=lambda k: sizes[k])
    near_1000 = sorted(range(len(sizes)), key=lambda k: abs(sizes[k] - 1000))[:2]
    odd = [k for k in by_size if wl.grids[k][0] % r or wl.grids[k][1] % r]
    square64 = [k for k in range(len(sizes)) if wl.grids[k] == (64, 64)]
    assert len(square64) == 1 and odd
    chosen = sorted(set(by_size[:3]) | set(near_1000) | {odd[-1]} | set(square64), key=lambda k: sizes[k])
    for i in chosen:
        sub = synth.Inputs(wl, synth.Tensor(inp.x.values[cu[i]:cu[i + 1]]), inp.layers, inp.final_norm_w,
                           inp.w_align)
        sub.wl = synth.Workload(wl.name, wl.dtype, wl.vision_dim, wl.n_heads, wl.mlp_hidden, r, wl.llm_dim,
                                wl.n_layers, [wl.grids[i]], wl.seed, True, True)
        t_o, a_o = O.encode(sub)
        e_t = rel_fro(tower_g[cu[i]:cu[i + 1]], t_o)
        e_a = rel_fro(align_g[tok[i]:tok[i + 1]], a_o)
        print(f"workload 5 image {i} {wl.grids[i]}: tower {e_t:.3e} aligner {e_a:.3e}")
        assert e_t <= 3e-2 and e_a <= 3e-2
    assert np.isfinite(tower_g).all() and np.isfinite(align_g).all()


# ------------------------------------------------------------------------------ boundary
def test_boundary_errors_on_device():
    wl = synth.workload(2)
    cfg = config_of(wl)
    b = A.BatchRef(wl.grids)
    n = A.dsv4v_workspace_size(cfg, b)
    small = torch.empty(n - 256, dtype=torch.uint8, device="cuda")
    x = torch.zeros(784, 1024, dtype=torch.bfloat16, device="cuda")
    cos = torch.zeros(784, 32, device="cuda")
    w = {k: torch.zeros(s, dtype=torch.bfloat16, device="cuda") for k, s in
         [("wqkv", (3072, 1024)), ("wo", (1024, 1024)), ("w_gate", (2816, 1024)), ("w_up", (2816, 1024)),
          ("w_down", (1024, 2816))]}
    w["norm1_w"] = torch.ones(1024, device="cuda")
    w["norm2_w"] = torch.ones(1024, device="cuda")
    bw = A.block_weights(w)
    with pytest.raises(A.Dsv4vError) as e:
        A.dsv4v_block_forward(cfg, b, bw, cos, cos, x, small)
    assert e.value.status == 3
    mis = torch.zeros(784 * 1024 + 8, dtype=torch.bfloat16, device="cuda")[1:1 + 784 * 1024]
    with pytest.raises(A.Dsv4vError) as e:
        A.dsv4v_block_forward(cfg, b, bw, cos, cos, mis, torch.empty(n, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 1
    # all-zero projections: the block is the identity (and nothing was launched by the failures)
    x0 = torch.randn(784, 1024, device="cuda").to(torch.bfloat16)
    x1 = x0.clone()
    A.dsv4v_block_forward(cfg, b, bw, cos, cos, x1, torch.empty(n, dtype=torch.uint8, device="cuda"))
    assert torch.equal(x0, x1)


def test_bounded_wait_records_timeout():
    assert A.dsv4v_device_error() == 0
    A.dsv4v_selftest_bounded_wait(2_000_000)  # 2 ms on a barrier nothing signals
    assert A.dsv4v_device_error() == 5        # DSV4V_ERR_TIMEOUT, recorded without a fault
    assert A.dsv4v_device_error() == 0        # and cleared
    x = torch.ones(4, device="cuda")
    assert float(x.sum()) == 4.0              # the context is still usable

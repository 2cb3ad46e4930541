"""The C-ABI library on a machine without a GPU: it builds, loads, exports every symbol the
header declares, and rejects bad arguments on the host before touching CUDA."""
import ctypes
import os
import re

import pytest

from vision_transformer_encoder_dsv4v_b200 import build
from vision_transformer_encoder_dsv4v_b200 import dsv4v as A

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return A.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "dsv4v.h")).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\**\s+\**(dsv4v_[a-z0-9_]+)\s*\(", text, re.M)))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 14, names
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(names) == sorted(A.EXPORTS)


def test_status_strings(lib):
    assert A.dsv4v_status_string(0) == "ok"
    assert "workspace" in A.dsv4v_status_string(3)
    assert A.dsv4v_status_string(99) == "unknown status"


class HostBatch:
    """A dsv4v_batch whose 'device' pointers are host buffers; only host validation reads them."""

    def __init__(self, grids, cu=None):
        self.grid = (ctypes.c_int32 * (2 * max(1, len(grids))))(*[v for g in grids for v in g])
        if cu is None:
            cu = [0]
            for h, w in grids:
                cu.append(cu[-1] + h * w)
        self.cu = (ctypes.c_int32 * len(cu))(*cu)
        self.c = A.Batch(len(grids), ctypes.addressof(self.grid), ctypes.addressof(self.grid),
                         ctypes.addressof(self.cu), ctypes.addressof(self.cu))


def cfg(**kw):
    d = dict(vision_dim=1024, n_heads=16, mlp_hidden=2816, downsample_ratio=2, llm_dim=4096, n_layers=32,
             dtype=A.DSV4V_BF16)
    d.update(kw)
    dt = d.pop("dtype")
    return A.make_config(dtype=dt, **d)


def test_workspace_size_and_tokens_host_only(lib):
    b = HostBatch([(28, 28)])
    n = lib.dsv4v_workspace_size(ctypes.byref(cfg()), ctypes.byref(b.c))
    # at least the activations: y, qkv, attn (bf16) and h, plus the rotary table
    assert n >= 784 * (1024 * 5 * 2 + 2816 * 2 + 32 * 8)
    assert lib.dsv4v_aligner_tokens(ctypes.byref(cfg()), ctypes.byref(b.c)) == 196
    b4 = HostBatch([(27, 37), (37, 27), (10, 78), (112, 7)])
    assert lib.dsv4v_aligner_tokens(ctypes.byref(cfg()), ctypes.byref(b4.c)) == 266 + 266 + 195 + 224


@pytest.mark.parametrize("case,status", [
    ("null_cfg", 1), ("zero_images", 1), ("bad_cu", 1), ("bad_cu0", 1), ("zero_side", 1),
    ("hd32_bf16", 2), ("dim_not_128", 2), ("hidden_not_128", 2), ("heads_not_dividing", 1), ("hd_odd_pairs", 2),
    ("f32_hd_too_big", 2), ("too_many_images", 1),
])
def test_host_validation_rejects(lib, case, status):
    c = cfg()
    b = HostBatch([(4, 6), (3, 5)])
    if case == "zero_images":
        b.c.n_images = 0
    elif case == "bad_cu":
        b = HostBatch([(4, 6), (3, 5)], cu=[0, 24, 40])
    elif case == "bad_cu0":
        b = HostBatch([(4, 6)], cu=[1, 25])
    elif case == "zero_side":
        b = HostBatch([(4, 0)])
    elif case == "hd32_bf16":
        c = cfg(n_heads=32)
    elif case == "dim_not_128":
        c = cfg(vision_dim=1088, n_heads=17)
    elif case == "hidden_not_128":
        c = cfg(mlp_hidden=2800)
    elif case == "heads_not_dividing":
        c = cfg(n_heads=15)
    elif case == "hd_odd_pairs":
        c = cfg(vision_dim=36, n_heads=6, dtype=A.DSV4V_F32)
    elif case == "f32_hd_too_big":
        c = cfg(vision_dim=256, n_heads=2, dtype=A.DSV4V_F32)
    elif case == "too_many_images":
        b = HostBatch([(1, 1)] * (A.DSV4V_MAX_IMAGES + 1))
    cp = None if case == "null_cfg" else ctypes.byref(c)
    x = ctypes.c_void_p(4096)
    w = A.BlockWeights(*([4096] * 7))
    st = lib.dsv4v_block_forward(cp, ctypes.byref(b.c), ctypes.byref(w), x, x, x, x, 1 << 30, None)
    assert st == status
    assert lib.dsv4v_workspace_size(cp, ctypes.byref(b.c)) == 0
    st = lib.dsv4v_aligner_forward(cp, ctypes.byref(b.c), x, x, x, None, x, 1 << 30, None)
    assert st == status


# ------------------------------------------------------------------------ image-token bridge
def test_image_layout_host_matches_oracle(lib):
    # the library's host N-layout against the oracle's, on the pages' grids and edge grids
    import numpy as np
    from oracle import dsv4v_oracle as O
    for n_h, n_w in [(28, 28), (27, 37), (37, 27), (10, 78), (112, 7), (1, 1), (1, 9), (9, 1)]:
        for r in (1, 2, 3, 4):
            np.testing.assert_array_equal(A.dsv4v_image_layout(n_h, n_w, r), O.image_layout(n_h, n_w, r))


def test_image_layout_argument_checks(lib):
    n = ctypes.c_int64(-1)
    assert lib.dsv4v_image_layout(0, 5, 2, None, 0, ctypes.byref(n)) == 1
    assert lib.dsv4v_image_layout(3, 5, 0, None, 0, ctypes.byref(n)) == 1
    assert lib.dsv4v_image_layout(3, 5, 2, None, 0, ctypes.byref(n)) == 0 and n.value == 10
    buf = (ctypes.c_int32 * 9)(*([77] * 9))
    assert lib.dsv4v_image_layout(3, 5, 2, ctypes.addressof(buf), 9, None) == 1  # too small
    assert list(buf) == [77] * 9  # nothing written


def test_bridge_workspace_size(lib):
    assert A.dsv4v_bridge_workspace_size(0) == 0
    assert A.dsv4v_bridge_workspace_size(1 << 31) == 0
    assert A.dsv4v_bridge_workspace_size(1) == 256 * 4  # counts + three int32 tables
    n = 256 * 16 + 1  # 17 chunks of counts (272 bytes -> 512), tables of 16388 bytes (-> 16640)
    assert A.dsv4v_bridge_workspace_size(n) == 512 + 3 * 16640


def test_bridge_host_validation_rejects(lib):
    # every rejection below happens on the host, before any CUDA call
    b = HostBatch([(3, 5)])
    c = cfg()
    al = 4096  # a 16-byte aligned fake address; never dereferenced
    ws = 1 << 20
    merge = lib.dsv4v_merge_image_embeddings
    assert merge(ctypes.byref(c), ctypes.byref(b.c), 0, 8, al, al, al, al, al, ws, None) == 1  # no sequences
    assert merge(ctypes.byref(c), ctypes.byref(b.c), 1, 8, None, al, al, al, al, ws, None) == 1  # no types
    assert merge(ctypes.byref(c), ctypes.byref(b.c), 1, 8, al, al + 8, al, al, al, ws, None) == 1  # misaligned
    assert merge(ctypes.byref(c), ctypes.byref(b.c), 1, 8, al, al, al, al, al, 0, None) == 3  # workspace
    assert merge(ctypes.byref(c), ctypes.byref(b.c), 1 << 20, 1 << 12, al, al, al, al, al, ws, None) == 1  # > 2^31
    f32 = cfg(dtype=A.DSV4V_F32, llm_dim=6, vision_dim=64, n_heads=4, mlp_hidden=96)
    assert merge(ctypes.byref(f32), ctypes.byref(b.c), 1, 8, al, al, al, al, al, ws, None) == 2  # 24-byte rows
    vis = lib.dsv4v_image_visibility
    assert vis(1, 8, al, al, 3, al, ws, None) == 1  # element size
    assert vis(1, 8, al, al + 2, 4, al, ws, None) == 1  # misaligned fp32 mask
    assert vis(0, 8, al, al, 4, al, ws, None) == 1
    assert vis(1, 8, None, al, 4, al, ws, None) == 1
    assert vis(1, 8, al, al, 4, al + 16, ws, None) == 3  # workspace not 256-byte aligned
    assert vis(1, 8, al, al, 4, al, 100, None) == 3  # workspace too small


def test_backward_host_checks(lib):
    # sizing is host-only; fp32 configs are rejected before any CUDA call
    b = HostBatch([(28, 28)])
    assert lib.dsv4v_backward_workspace_size(ctypes.byref(cfg()), ctypes.byref(b.c)) > 0
    f32 = cfg(dtype=A.DSV4V_F32, vision_dim=64, n_heads=4, mlp_hidden=128, llm_dim=128)
    assert lib.dsv4v_backward_workspace_size(ctypes.byref(f32), ctypes.byref(b.c)) == 0
    assert lib.dsv4v_attention_backward(ctypes.byref(f32), ctypes.byref(b.c), None, None, None, None, None, 0,
                                        None) == 2
    assert lib.dsv4v_block_backward(ctypes.byref(f32), ctypes.byref(b.c), None, None, None, None, None, None, None,
                                    None, 0, None) == 2
    # the scratch grows with the patches: every activation and gradient of the block is kept
    small = lib.dsv4v_backward_workspace_size(ctypes.byref(cfg()), ctypes.byref(HostBatch([(3, 5)]).c))
    big = lib.dsv4v_backward_workspace_size(ctypes.byref(cfg()), ctypes.byref(b.c))
    assert 0 < small < big


def test_header_compiles_as_c99_and_links(lib, tmp_path):
    # the public header is plain C: a C99 program includes it, links the library and runs the
    # calls that need no GPU
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    exe = tmp_path / "abi_host_check"
    libdir = os.path.dirname(A.LIB_PATH)
    subprocess.run([cc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", os.path.join(ROOT, "include"),
                    os.path.join(ROOT, "tests", "c", "abi_host_check.c"), "-o", str(exe), "-L", libdir, "-ldsv4v",
                    f"-Wl,-rpath,{libdir}"], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    assert "c abi ok" in r.stdout


def test_tower_path_choice_and_validation():
    """The launch-sequence setting and its automatic choice (host logic only: no kernel runs)."""
    from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
    try:
        with pytest.raises(A.Dsv4vError):
            A.dsv4v_set_tower_path(7)
        cfg = A.make_config(1024, 16, 2816, 2, 4096, 1)
        A.dsv4v_set_tower_path(A.PATH_AUTO)
        assert A.dsv4v_tower_path(cfg, A.BatchRef([(64, 64), (8, 8)], device=None)) == A.PATH_KERNELS
        A.dsv4v_set_tower_path(A.PATH_KERNELS)
        assert A.dsv4v_tower_path(cfg, A.BatchRef([(28, 28)], device=None)) == A.PATH_KERNELS
        A.dsv4v_set_tower_path(A.PATH_CHAIN)
        assert A.dsv4v_tower_path(cfg, A.BatchRef([(64, 64), (8, 8)], device=None)) == A.PATH_CHAIN
        cfg32 = A.make_config(64, 4, 128, 2, 128, 1, dtype=A.DSV4V_F32)
        assert A.dsv4v_tower_path(cfg32, A.BatchRef([(4, 6)], device=None)) == A.PATH_KERNELS
    finally:
        A.dsv4v_set_tower_path(A.PATH_AUTO)


def test_graph_replay_switch_needs_no_gpu():
    """The step calls' graph-replay switch and the release of the calling thread's cached
    executables are host state only: both run without a GPU, repeatedly, and in any order."""
    from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
    for _ in range(2):
        A.dsv4v_release_graphs()
        A.dsv4v_set_graph_replay(False)
        A.dsv4v_release_graphs()
        A.dsv4v_set_graph_replay(True)


def test_step_launch_count():
    """The per-step launch count the benchmark reports: rotary table, first norm operand, per
    layer 4 GEMMs + attention (or attention + one chain launch), final norm, aligner (window
    index, merged rows, GEMM)."""
    from vision_transformer_encoder_dsv4v_b200 import dsv4v as A
    cfg = A.make_config(1024, 16, 2816, 2, 4096, 32)
    one = A.BatchRef([(28, 28)], device=None)
    try:
        A.dsv4v_set_tower_path(A.PATH_KERNELS)
        assert A.dsv4v_step_launches(cfg, one) == 1 + 1 + 5 * 32 + 1 + 3
        assert A.dsv4v_step_launches(cfg, one, final_norm=False, aligner=False) == 1 + 1 + 5 * 32
        A.dsv4v_set_tower_path(A.PATH_CHAIN)
        assert A.dsv4v_step_launches(cfg, one) == 1 + 2 + 2 * 32 + 1 + 3
    finally:
        A.dsv4v_set_tower_path(A.PATH_AUTO)
    with pytest.raises(A.Dsv4vError):
        A.dsv4v_step_launches(cfg, A.BatchRef([(0, 3)], device=None))

"""Python binding of the dsv4v C ABI (include/dsv4v.h): argument marshalling only.

Every function here has the name of the C entry point it calls and passes raw device pointers
of torch tensors plus the current CUDA stream; all arithmetic happens in the CUDA library.
There is no fallback: if ``libdsv4v.so`` cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libdsv4v.so")

DSV4V_F32 = 0
DSV4V_BF16 = 1
DSV4V_MAX_IMAGES = 1024

STATUS = {0: "DSV4V_OK", 1: "DSV4V_ERR_INVALID_ARG", 2: "DSV4V_ERR_UNSUPPORTED", 3: "DSV4V_ERR_WORKSPACE",
          4: "DSV4V_ERR_CUDA", 5: "DSV4V_ERR_TIMEOUT", 6: "DSV4V_ERR_LAYOUT"}
DSV4V_ERR_INVALID_ARG = 1
DSV4V_ERR_TIMEOUT = 5
DSV4V_ERR_LAYOUT = 6

# Pseudo-token types of the image-token bridge (DSV4V_TOKEN_*); sentinel rows follow types 1..4.
TOKEN_TEXT, TOKEN_IMAGE, TOKEN_START, TOKEN_END, TOKEN_NEWLINE, TOKEN_PAD = -1, 0, 1, 2, 3, 4

PROFILE_KINDS = ("qkv", "attention", "out", "swiglu", "down", "chain")  # DSV4V_PROFILE_* order

# Launch sequences of the bf16 blocks (DSV4V_PATH_*).
PATH_AUTO, PATH_KERNELS, PATH_CHAIN = 0, 1, 2

# Every symbol include/dsv4v.h declares.
EXPORTS = ("dsv4v_workspace_size", "dsv4v_rope2d_table", "dsv4v_block_forward", "dsv4v_tower_forward",
           "dsv4v_tower_forward_profiled",
           "dsv4v_aligner_forward", "dsv4v_aligner_tokens", "dsv4v_rmsnorm", "dsv4v_qkv_rope", "dsv4v_attention",
           "dsv4v_linear_residual", "dsv4v_swiglu", "dsv4v_device_error", "dsv4v_selftest_bounded_wait",
           "dsv4v_status_string", "dsv4v_linear_residual_noalloc", "dsv4v_patch_embed",
           "dsv4v_patch_merger_workspace_size", "dsv4v_patch_merger_forward", "dsv4v_image_layout",
           "dsv4v_bridge_workspace_size", "dsv4v_merge_image_embeddings", "dsv4v_image_visibility",
           "dsv4v_backward_workspace_size", "dsv4v_attention_backward", "dsv4v_rmsnorm_backward",
           "dsv4v_block_backward", "dsv4v_tower_backward", "dsv4v_set_tower_path", "dsv4v_tower_path",
           "dsv4v_step_launches", "dsv4v_set_graph_replay", "dsv4v_release_graphs")

DSV4V_NOALLOC_MAX_ROWS = 65536


class Dsv4vError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


class Config(ctypes.Structure):
    _fields_ = [("vision_dim", ctypes.c_int), ("n_heads", ctypes.c_int), ("mlp_hidden", ctypes.c_int),
                ("downsample_ratio", ctypes.c_int), ("llm_dim", ctypes.c_int), ("n_layers", ctypes.c_int),
                ("eps", ctypes.c_float), ("rope_theta", ctypes.c_float), ("dtype", ctypes.c_int)]


class BlockWeights(ctypes.Structure):
    _fields_ = [("norm1_w", ctypes.c_void_p), ("norm2_w", ctypes.c_void_p), ("wqkv", ctypes.c_void_p),
                ("wo", ctypes.c_void_p), ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p)]


class BlockGrads(ctypes.Structure):
    _fields_ = [("norm1_w", ctypes.c_void_p), ("norm2_w", ctypes.c_void_p), ("wqkv", ctypes.c_void_p),
                ("wo", ctypes.c_void_p), ("w_gate", ctypes.c_void_p), ("w_up", ctypes.c_void_p),
                ("w_down", ctypes.c_void_p)]


class Batch(ctypes.Structure):
    _fields_ = [("n_images", ctypes.c_int), ("grid_hw_host", ctypes.c_void_p), ("grid_hw_dev", ctypes.c_void_p),
                ("cu_patches_host", ctypes.c_void_p), ("cu_patches_dev", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Loads libdsv4v.so (built by ``build.build()``); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run vision_transformer_encoder_dsv4v_b200.build.build()")
        L = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64
        cfg, bat, bw = ctypes.POINTER(Config), ctypes.POINTER(Batch), ctypes.POINTER(BlockWeights)
        sig = {
            "dsv4v_workspace_size": (SZ, [cfg, bat]),
            "dsv4v_aligner_tokens": (I64, [cfg, bat]),
            "dsv4v_rope2d_table": (I, [cfg, bat, P, P, P]),
            "dsv4v_block_forward": (I, [cfg, bat, bw, P, P, P, P, SZ, P]),
            "dsv4v_tower_forward": (I, [cfg, bat, bw, P, P, P, SZ, P]),
            "dsv4v_tower_forward_profiled": (I, [cfg, bat, bw, P, P, P, SZ, P, P]),
            "dsv4v_aligner_forward": (I, [cfg, bat, P, P, P, P, P, SZ, P]),
            "dsv4v_rmsnorm": (I, [cfg, I64, P, P, P, P]),
            "dsv4v_qkv_rope": (I, [cfg, bat, P, P, P, P, P, P, SZ, P]),
            "dsv4v_attention": (I, [cfg, bat, P, P, P]),
            "dsv4v_linear_residual": (I, [cfg, I64, I, P, P, P, P, SZ, P]),
            "dsv4v_swiglu": (I, [cfg, I64, P, P, P, P, P, SZ, P]),
            "dsv4v_patch_embed": (I, [cfg, I64, I, I, P, I64, P, I64, P, P, P]),
            "dsv4v_patch_merger_workspace_size": (SZ, [cfg, bat]),
            "dsv4v_patch_merger_forward": (I, [cfg, bat, P, P, P, P, P, P, P, P, P, SZ, P]),
            "dsv4v_linear_residual_noalloc": (I, [cfg, I64, I, P, P, P, P]),
            "dsv4v_image_layout": (I, [I, I, I, P, I64, ctypes.POINTER(ctypes.c_int64)]),
            "dsv4v_backward_workspace_size": (SZ, [cfg, bat]),
            "dsv4v_attention_backward": (I, [cfg, bat, P, P, P, P, P, SZ, P]),
            "dsv4v_rmsnorm_backward": (I, [cfg, bat, P, P, P, P, P, P, P, SZ, P]),
            "dsv4v_block_backward": (I, [cfg, bat, bw, P, P, P, P, P, ctypes.POINTER(BlockGrads), P, SZ, P]),
            "dsv4v_tower_backward": (I, [cfg, bat, bw, P, P, P, P, P, ctypes.POINTER(BlockGrads), P, P, SZ, P]),
            "dsv4v_bridge_workspace_size": (SZ, [I64]),
            "dsv4v_merge_image_embeddings": (I, [cfg, bat, I64, I64, P, P, P, P, P, SZ, P]),
            "dsv4v_image_visibility": (I, [I64, I64, P, P, I, P, SZ, P]),
            "dsv4v_device_error": (I, [P]),
            "dsv4v_selftest_bounded_wait": (I, [U64, P]),
            "dsv4v_status_string": (ctypes.c_char_p, [I]),
            "dsv4v_set_tower_path": (I, [I]),
            "dsv4v_tower_path": (I, [cfg, bat]),
            "dsv4v_step_launches": (I, [cfg, bat, I, I]),
            "dsv4v_set_graph_replay": (None, [I]),
            "dsv4v_release_graphs": (None, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


# ------------------------------------------------------------------------------ marshalling
def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is not None:
        return ctypes.c_void_p(stream)
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _check(status: int, where: str):
    if status != 0:
        raise Dsv4vError(status, where)


def make_config(vision_dim, n_heads, mlp_hidden, downsample_ratio, llm_dim, n_layers, eps=1e-6, rope_theta=10000.0,
                dtype=DSV4V_BF16) -> Config:
    return Config(vision_dim, n_heads, mlp_hidden, downsample_ratio, llm_dim, n_layers, eps, rope_theta, dtype)


class BatchRef:
    """A dsv4v_batch plus the host and device int32 tensors it points to (kept alive here)."""

    def __init__(self, grids, device="cuda"):
        import torch
        self.grids = [(int(h), int(w)) for h, w in grids]
        cu = [0]
        for h, w in self.grids:
            cu.append(cu[-1] + h * w)
        self.grid_host = torch.tensor(self.grids, dtype=torch.int32).reshape(-1, 2).contiguous()
        self.cu_host = torch.tensor(cu, dtype=torch.int32)
        self.grid_dev = self.grid_host.to(device)
        self.cu_dev = self.cu_host.to(device)
        self.n_patches = cu[-1]
        self.c = Batch(len(self.grids), self.grid_host.data_ptr(), self.grid_dev.data_ptr(), self.cu_host.data_ptr(),
                       self.cu_dev.data_ptr())


def block_weights(layer: dict) -> BlockWeights:
    """layer: dict of device tensors norm1_w, norm2_w (fp32) and wqkv, wo, w_gate, w_up, w_down."""
    return BlockWeights(*(layer[k].data_ptr() for k in ("norm1_w", "norm2_w", "wqkv", "wo", "w_gate", "w_up", "w_down")))


# ------------------------------------------------------------------------------ entry points
def dsv4v_workspace_size(cfg: Config, batch: BatchRef) -> int:
    return int(lib().dsv4v_workspace_size(ctypes.byref(cfg), ctypes.byref(batch.c)))


def dsv4v_aligner_tokens(cfg: Config, batch: BatchRef) -> int:
    return int(lib().dsv4v_aligner_tokens(ctypes.byref(cfg), ctypes.byref(batch.c)))


def dsv4v_rope2d_table(cfg, batch, cos_out, sin_out, stream=None):
    _check(lib().dsv4v_rope2d_table(ctypes.byref(cfg), ctypes.byref(batch.c), _ptr(cos_out), _ptr(sin_out),
                                    _stream(stream)), "dsv4v_rope2d_table")


def dsv4v_block_forward(cfg, batch, weights: BlockWeights, cos, sin, x_inout, workspace, stream=None):
    _check(lib().dsv4v_block_forward(ctypes.byref(cfg), ctypes.byref(batch.c), ctypes.byref(weights), _ptr(cos),
                                     _ptr(sin), _ptr(x_inout), _ptr(workspace), workspace.numel(), _stream(stream)),
           "dsv4v_block_forward")


def dsv4v_tower_forward(cfg, batch, layers, final_norm_w, x_inout, workspace, stream=None):
    arr = (BlockWeights * max(1, len(layers)))(*layers)
    _check(lib().dsv4v_tower_forward(ctypes.byref(cfg), ctypes.byref(batch.c), arr, _ptr(final_norm_w),
                                     _ptr(x_inout), _ptr(workspace), workspace.numel(), _stream(stream)),
           "dsv4v_tower_forward")


def dsv4v_set_graph_replay(enable):
    """Process-wide switch of the step calls' graph replay (on by default): repeated
    dsv4v_tower_forward / dsv4v_aligner_forward calls with identical arguments on a non-default
    stream replay a CUDA graph captured on the second such call."""
    lib().dsv4v_set_graph_replay(1 if enable else 0)


def dsv4v_release_graphs():
    """Destroys every cached graph executable of the step calls."""
    lib().dsv4v_release_graphs()


def dsv4v_set_tower_path(path):
    """Process-wide choice of the bf16 blocks' launch sequence (PATH_AUTO, PATH_KERNELS or
    PATH_CHAIN) for the calls that follow; size workspaces after setting it."""
    _check(lib().dsv4v_set_tower_path(int(path)), "dsv4v_set_tower_path")


def dsv4v_tower_path(cfg, batch):
    """PATH_KERNELS or PATH_CHAIN: the sequence the block and tower calls use for this batch."""
    r = lib().dsv4v_tower_path(ctypes.byref(cfg), ctypes.byref(batch.c))
    if r < 0:
        raise Dsv4vError(DSV4V_ERR_INVALID_ARG, "dsv4v_tower_path")
    return r


def dsv4v_step_launches(cfg, batch, final_norm=True, aligner=True):
    """Kernel launches of dsv4v_tower_forward (+ final norm) followed by dsv4v_aligner_forward."""
    r = lib().dsv4v_step_launches(ctypes.byref(cfg), ctypes.byref(batch.c), int(bool(final_norm)), int(bool(aligner)))
    if r < 0:
        raise Dsv4vError(DSV4V_ERR_INVALID_ARG, "dsv4v_step_launches")
    return r


def dsv4v_tower_forward_profiled(cfg, batch, layers, final_norm_w, x_inout, workspace, events, stream=None):
    """events: sequence of n_layers * len(PROFILE_KINDS) * 2 torch.cuda.Event (or None), already
    recorded once so that their CUDA handles exist; [(layer * kinds + kind) * 2 + 0/1]."""
    arr = (BlockWeights * max(1, len(layers)))(*layers)
    handles = (ctypes.c_void_p * len(events))(*[(e.cuda_event if e is not None else None) for e in events])
    _check(lib().dsv4v_tower_forward_profiled(ctypes.byref(cfg), ctypes.byref(batch.c), arr, _ptr(final_norm_w),
                                              _ptr(x_inout), _ptr(workspace), workspace.numel(), _stream(stream),
                                              handles), "dsv4v_tower_forward_profiled")


def dsv4v_aligner_forward(cfg, batch, x, w_align, out, workspace, cu_tokens_host=None, stream=None):
    buf = None
    if cu_tokens_host is not None:
        buf = cu_tokens_host.data_ptr()
    _check(lib().dsv4v_aligner_forward(ctypes.byref(cfg), ctypes.byref(batch.c), _ptr(x), _ptr(w_align), _ptr(out),
                                       buf, _ptr(workspace), workspace.numel(), _stream(stream)),
           "dsv4v_aligner_forward")


def dsv4v_rmsnorm(cfg, rows, x, w, y, stream=None):
    _check(lib().dsv4v_rmsnorm(ctypes.byref(cfg), rows, _ptr(x), _ptr(w), _ptr(y), _stream(stream)), "dsv4v_rmsnorm")


def dsv4v_qkv_rope(cfg, batch, y, wqkv, cos, sin, qkv, workspace, stream=None):
    _check(lib().dsv4v_qkv_rope(ctypes.byref(cfg), ctypes.byref(batch.c), _ptr(y), _ptr(wqkv), _ptr(cos), _ptr(sin),
                                _ptr(qkv), _ptr(workspace), workspace.numel(), _stream(stream)), "dsv4v_qkv_rope")


def dsv4v_attention(cfg, batch, qkv, out, stream=None):
    _check(lib().dsv4v_attention(ctypes.byref(cfg), ctypes.byref(batch.c), _ptr(qkv), _ptr(out), _stream(stream)),
           "dsv4v_attention")


def dsv4v_linear_residual(cfg, rows, k, a, w, x, workspace, stream=None):
    _check(lib().dsv4v_linear_residual(ctypes.byref(cfg), rows, k, _ptr(a), _ptr(w), _ptr(x), _ptr(workspace),
                                       workspace.numel() if workspace is not None else 0, _stream(stream)),
           "dsv4v_linear_residual")


def dsv4v_linear_residual_noalloc(cfg, rows, k, a, w, x, stream=None):
    """x <- x + a . w^T with no workspace: for callers that cannot allocate device memory (the
    library's own static scratch is used; see include/dsv4v.h)."""
    _check(lib().dsv4v_linear_residual_noalloc(ctypes.byref(cfg), rows, k, _ptr(a), _ptr(w), _ptr(x), _stream(stream)),
           "dsv4v_linear_residual_noalloc")


def dsv4v_swiglu(cfg, rows, y, w_gate, w_up, h, workspace, stream=None):
    _check(lib().dsv4v_swiglu(ctypes.byref(cfg), rows, _ptr(y), _ptr(w_gate), _ptr(w_up), _ptr(h), _ptr(workspace),
                              workspace.numel() if workspace is not None else 0, _stream(stream)), "dsv4v_swiglu")


def dsv4v_patch_embed(cfg, n_patches, patch_h, patch_w, patches, w_proj, bias, x_out, ld_patches=0, ld_w=0,
                      stream=None):
    """x_out = patches . w_proj^T (+ bias): rows of `patches` are flattened (3, patch_h, patch_w)
    patches with row stride ld_patches (0: 3 * patch_h * patch_w); w_proj rows have stride ld_w."""
    _check(lib().dsv4v_patch_embed(ctypes.byref(cfg), n_patches, patch_h, patch_w, _ptr(patches), ld_patches,
                                   _ptr(w_proj), ld_w, _ptr(bias), _ptr(x_out), _stream(stream)),
           "dsv4v_patch_embed")


def dsv4v_patch_merger_workspace_size(cfg, batch) -> int:
    return int(lib().dsv4v_patch_merger_workspace_size(ctypes.byref(cfg), ctypes.byref(batch.c)))


def dsv4v_patch_merger_forward(cfg, batch, x, ln_w, ln_b, w1, b1, w2, b2, out, workspace, stream=None):
    """PatchMerger projector: LayerNorm per patch, r x r window merge, Linear + GELU, Linear."""
    _check(lib().dsv4v_patch_merger_forward(ctypes.byref(cfg), ctypes.byref(batch.c), _ptr(x), _ptr(ln_w), _ptr(ln_b),
                                            _ptr(w1), _ptr(b1), _ptr(w2), _ptr(b2), _ptr(out), _ptr(workspace),
                                            workspace.numel() if workspace is not None else 0, _stream(stream)),
           "dsv4v_patch_merger_forward")


def dsv4v_image_layout(grid_h: int, grid_w: int, downsample_ratio: int):
    """N-layout of one image as a host numpy int32 array (computed by the C library)."""
    import numpy as np
    n = ctypes.c_int64(0)
    _check(lib().dsv4v_image_layout(grid_h, grid_w, downsample_ratio, None, 0, ctypes.byref(n)), "dsv4v_image_layout")
    out = np.empty(n.value, dtype=np.int32)
    _check(lib().dsv4v_image_layout(grid_h, grid_w, downsample_ratio, out.ctypes.data_as(ctypes.c_void_p), n.value,
                                    None), "dsv4v_image_layout")
    return out


def dsv4v_bridge_workspace_size(n_positions: int) -> int:
    return int(lib().dsv4v_bridge_workspace_size(n_positions))


def dsv4v_merge_image_embeddings(cfg, batch, token_types, image_tokens, sentinels, embeds, workspace, stream=None):
    """embeds [n_seqs, seq_len, E] (updated in place) <- image tokens and sentinels at the
    pseudo-token positions of token_types [n_seqs, seq_len] (int32)."""
    n_seqs, seq_len = int(embeds.shape[0]), int(embeds.shape[1])
    _check(lib().dsv4v_merge_image_embeddings(ctypes.byref(cfg), ctypes.byref(batch.c), n_seqs, seq_len,
                                              _ptr(token_types), _ptr(image_tokens), _ptr(sentinels), _ptr(embeds),
                                              _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                              _stream(stream)),
           "dsv4v_merge_image_embeddings")


def dsv4v_image_visibility(token_types, mask, workspace, stream=None):
    """mask [n_seqs, seq_len, seq_len] (or with a unit head axis), updated in place: every pair
    inside one image span of token_types [n_seqs, seq_len] becomes 0."""
    n_seqs, seq_len = int(token_types.shape[0]), int(token_types.shape[1])
    if mask.numel() != n_seqs * seq_len * seq_len:
        raise ValueError(f"mask has {mask.numel()} entries, expected {n_seqs} x {seq_len} x {seq_len}")
    _check(lib().dsv4v_image_visibility(n_seqs, seq_len, _ptr(token_types), _ptr(mask), mask.element_size(),
                                        _ptr(workspace), workspace.numel() if workspace is not None else 0,
                                        _stream(stream)),
           "dsv4v_image_visibility")


# ------------------------------------------------------------------------------ backward
def block_grads(norm1_w, norm2_w, wqkv, wo, w_gate, w_up, w_down) -> BlockGrads:
    """A dsv4v_block_grads of the given device tensors (the caller keeps them alive)."""
    return BlockGrads(*[t.data_ptr() for t in (norm1_w, norm2_w, wqkv, wo, w_gate, w_up, w_down)])


def dsv4v_backward_workspace_size(cfg, batch) -> int:
    return int(lib().dsv4v_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(batch.c)))


def _ws(workspace):
    return _ptr(workspace), workspace.numel() if workspace is not None else 0


def dsv4v_attention_backward(cfg, batch, qkv, out, d_out, dqkv, workspace, stream=None):
    """dqkv [P, 3D] <- gradients of the attention w.r.t. its (rotated) q, k and v."""
    _check(lib().dsv4v_attention_backward(ctypes.byref(cfg), ctypes.byref(batch.c), _ptr(qkv), _ptr(out), _ptr(d_out),
                                          _ptr(dqkv), *_ws(workspace), _stream(stream)),
           "dsv4v_attention_backward")


def dsv4v_rmsnorm_backward(cfg, batch, x, w, dy, d_in, dx, dw, workspace, stream=None):
    _check(lib().dsv4v_rmsnorm_backward(ctypes.byref(cfg), ctypes.byref(batch.c), _ptr(x), _ptr(w), _ptr(dy),
                                        _ptr(d_in), _ptr(dx), _ptr(dw), *_ws(workspace), _stream(stream)),
           "dsv4v_rmsnorm_backward")


def dsv4v_block_backward(cfg, batch, weights, cos, sin, x, d_out, dx, grads, workspace, stream=None):
    """weights: BlockWeights; grads: BlockGrads (see block_grads)."""
    _check(lib().dsv4v_block_backward(ctypes.byref(cfg), ctypes.byref(batch.c), ctypes.byref(weights), _ptr(cos),
                                      _ptr(sin), _ptr(x), _ptr(d_out), _ptr(dx), ctypes.byref(grads), *_ws(workspace),
                                      _stream(stream)),
           "dsv4v_block_backward")


def dsv4v_tower_backward(cfg, batch, layers, final_norm_w, layer_inputs, x_last, d_out, dx, layer_grads,
                         d_final_norm_w, workspace, stream=None):
    """layers: list of BlockWeights; layer_inputs: list of device tensors (each block's input);
    layer_grads: list of BlockGrads."""
    n = len(layer_inputs)
    arr = (BlockWeights * n)(*layers)
    inputs = (ctypes.c_void_p * n)(*[t.data_ptr() for t in layer_inputs])
    grads = (BlockGrads * n)(*layer_grads)
    _check(lib().dsv4v_tower_backward(ctypes.byref(cfg), ctypes.byref(batch.c), arr, _ptr(final_norm_w), inputs,
                                      _ptr(x_last), _ptr(d_out), _ptr(dx), grads, _ptr(d_final_norm_w),
                                      *_ws(workspace), _stream(stream)),
           "dsv4v_tower_backward")


def dsv4v_device_error(stream=None) -> int:
    return int(lib().dsv4v_device_error(_stream(stream)))


def dsv4v_selftest_bounded_wait(limit_ns: int, stream=None):
    _check(lib().dsv4v_selftest_bounded_wait(limit_ns, _stream(stream)), "dsv4v_selftest_bounded_wait")


def dsv4v_status_string(status: int) -> str:
    return lib().dsv4v_status_string(status).decode()

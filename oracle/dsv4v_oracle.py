"""fp64 CPU oracle of the DeepSeek-V4-Flash vision tower forward pass.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's CPU-baseline leg
may import this module.  The CUDA library never calls it, and it imports nothing from the CUDA
path: it is a plain, slow restatement of what the pages define, in float64, with numpy's matmul
as the only library primitive.  No blocking, fusion or reordering beyond the definitions.

Sources (page title, then section):
  [vision-API]  "nemo_automodel.components.models.deepseek_v4.vision" API reference
                (classes DeepseekV4VisionRMSNorm / Attention / MLP / Block / Transformer /
                Aligner, functions apply_vision_rotary, get_vision_cos_sin)
  [model-API]   "nemo_automodel.components.models.deepseek_v4.model" API reference
                (DeepseekV4Model.encode_image, merge_image_embeddings and the sentinel
                parameters image_start / image_end / image_newline / image_pad,
                apply_deepseek_v4_image_visibility, the THD cu_seqlens helpers)
  [PR]          NeMo-Automodel pull request "Add native AutoModel support for
                deepseek-ai/DeepSeek-V4-Flash-Vision-Exp", Changelog and Validation

Where the pages leave a step open the function says "READING n"; the design notes list every
reading.  Every function is pinned by the not-gpu tests (closed forms, invariants, brute force
on tiny inputs, a hand-written aligner table) -- none is "parity unpinned" except that the
*choice* among the readings themselves cannot be pinned without the released weights.

Layouts: activations are packed varlen ``[P, D]`` (all images' patches back to back, patch
``p = h * n_w + w`` row-major inside an image, READING 12); ``grids`` is a list of (n_h, n_w);
weights are ``[out, in]``.
"""
from __future__ import annotations

import math

import numpy as np


def _f64(a) -> np.ndarray:
    return np.asarray(a, dtype=np.float64)


def cu_from_grids(grids) -> np.ndarray:
    """Packed varlen offsets in the cu_seqlens form of [model-API, THD packing helpers]:
    length n_images + 1, starting at 0, entry i+1 - entry i = n_h * n_w of image i."""
    cu = [0]
    for n_h, n_w in grids:
        cu.append(cu[-1] + n_h * n_w)
    return np.asarray(cu, dtype=np.int64)


# --------------------------------------------------------------------------------------------
# RMSNorm  [vision-API, DeepseekV4VisionRMSNorm]: RMSNorm over the last axis with an fp32
# scale parameter, eps default 1e-6.  READING 3: y = w * x / sqrt(mean(x^2) + eps), with the
# weight applied directly (not 1 + w).
# --------------------------------------------------------------------------------------------
def rmsnorm(x, weight, eps: float = 1e-6) -> np.ndarray:
    x = _f64(x)
    mean_sq = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(mean_sq + eps) * _f64(weight)


# --------------------------------------------------------------------------------------------
# 2D rotary table  [vision-API, get_vision_cos_sin]: the table for an n_h x n_w patch grid,
# layout [n_h*n_w, 1, dim] on the page; the singleton head axis is dropped here.
# READING 2: dim = head_dim / 2 (the table is what apply_vision_rotary consumes, whose cos/sin
# layout is [patches, 1, head_dim/2]).
# READING 1: the first dim/2 angles rotate by the patch's row index, the last dim/2 by its
# column index; both halves share inv_freq_k = theta ** (-k / (dim/2)), k < dim/2; positions are
# the integer grid coordinates of the patch inside its own image, starting at 0.
# --------------------------------------------------------------------------------------------
def vision_cos_sin(n_h: int, n_w: int, dim: int, theta: float):
    if dim % 2:
        raise ValueError("the 2D table needs an even width (head_dim % 4 == 0)")
    quarter = dim // 2
    inv_freq = np.asarray([theta ** (-k / quarter) for k in range(quarter)], dtype=np.float64)
    angles = np.zeros((n_h * n_w, dim), dtype=np.float64)
    for h in range(n_h):
        for w in range(n_w):
            p = h * n_w + w
            angles[p, :quarter] = h * inv_freq
            angles[p, quarter:] = w * inv_freq
    return np.cos(angles), np.sin(angles)


def packed_cos_sin(grids, dim: int, theta: float):
    """Per-image tables stacked in packing order: row p of the result belongs to the patch in
    row p of the packed activations (each image restarts at position (0, 0))."""
    cs = [vision_cos_sin(h, w, dim, theta) for h, w in grids]
    return np.concatenate([c for c, _ in cs]), np.concatenate([s for _, s in cs])


# --------------------------------------------------------------------------------------------
# Half-split rotation  [vision-API, apply_vision_rotary]: x [patches, heads, head_dim],
# cos/sin [patches, 1, head_dim/2].  "Half-split": channel j pairs with channel j + head_dim/2
# (the rotate-half convention); the pair is rotated by the angle of column j of the table.
# --------------------------------------------------------------------------------------------
def apply_vision_rotary(x, cos, sin) -> np.ndarray:
    x = _f64(x)
    half = x.shape[-1] // 2
    c = _f64(cos)[:, None, :]
    s = _f64(sin)[:, None, :]
    first, second = x[..., :half], x[..., half:]
    return np.concatenate([first * c - second * s, second * c + first * s], axis=-1)


# --------------------------------------------------------------------------------------------
# Attention  [vision-API, DeepseekV4VisionAttention / DeepseekV4VisionTransformer]: "full
# bidirectional patch attention", "full attention over one image".  READING 6: scale
# 1/sqrt(head_dim), no mask, no bias, no sinks.  READING 11: images of a packed batch never
# attend to each other.
# --------------------------------------------------------------------------------------------
def attention_probs(q, k) -> np.ndarray:
    """softmax(q k^T / sqrt(hd)) for one image and one head; q, k [N, hd] -> [N, N]."""
    q, k = _f64(q), _f64(k)
    scores = q @ k.T / math.sqrt(q.shape[-1])
    scores = scores - scores.max(axis=1, keepdims=True)
    e = np.exp(scores)
    return e / e.sum(axis=1, keepdims=True)


def attention_one_image(q, k, v) -> np.ndarray:
    """q, k, v [N, H, hd] of one image -> [N, H*hd], heads concatenated in head order
    (READING 5)."""
    n, n_heads, hd = q.shape
    out = np.zeros((n, n_heads, hd), dtype=np.float64)
    for h in range(n_heads):
        out[:, h, :] = attention_probs(q[:, h, :], k[:, h, :]) @ _f64(v[:, h, :])
    return out.reshape(n, n_heads * hd)


def attention_packed(q, k, v, grids) -> np.ndarray:
    cu = cu_from_grids(grids)
    return np.concatenate([attention_one_image(q[a:b], k[a:b], v[a:b])
                           for a, b in zip(cu[:-1], cu[1:])])


# --------------------------------------------------------------------------------------------
# SwiGLU MLP  [vision-API, DeepseekV4VisionMLP]: "bias-free SwiGLU", [P, D] -> [P, D].
# READING 7: silu(y Wg^T) * (y Wu^T), then Wd; silu(z) = z / (1 + exp(-z)); no clamp.
# --------------------------------------------------------------------------------------------
def silu(z) -> np.ndarray:
    z = _f64(z)
    return z / (1.0 + np.exp(-z))


def mlp(y, w_gate, w_up, w_down) -> np.ndarray:
    y = _f64(y)
    return (silu(y @ _f64(w_gate).T) * (y @ _f64(w_up).T)) @ _f64(w_down).T


def qkv_rope(y, wqkv, cos, sin, n_heads: int):
    """The fused projection [vision-API, DeepseekV4VisionAttention.wqkv] followed by the
    rotation of q and k.  READING 5: rows of wqkv are q | k | v blocks of D rows, head-major
    inside each block.  READING 4: no bias.  Returns q, k, v as [P, H, hd]."""
    y = _f64(y)
    d = y.shape[1]
    hd = d // n_heads
    qkv = y @ _f64(wqkv).T
    q = qkv[:, :d].reshape(-1, n_heads, hd)
    k = qkv[:, d:2 * d].reshape(-1, n_heads, hd)
    v = qkv[:, 2 * d:].reshape(-1, n_heads, hd)
    return apply_vision_rotary(q, cos, sin), apply_vision_rotary(k, cos, sin), v


# --------------------------------------------------------------------------------------------
# Block  [vision-API, DeepseekV4VisionBlock]: pre-norm attention and MLP residual block,
# x + attn(norm1(x)), then x + mlp(norm2(x)).  The output projection after attention has no
# name on the pages (READING 4: bias-free, weight wo [D, D]).
# --------------------------------------------------------------------------------------------
def block_forward(x, layer: dict, cos, sin, grids, n_heads: int, eps: float = 1e-6) -> np.ndarray:
    x = _f64(x)
    y = rmsnorm(x, layer["norm1_w"], eps)
    q, k, v = qkv_rope(y, layer["wqkv"], cos, sin, n_heads)
    x = x + attention_packed(q, k, v, grids) @ _f64(layer["wo"]).T
    y = rmsnorm(x, layer["norm2_w"], eps)
    return x + mlp(y, layer["w_gate"], layer["w_up"], layer["w_down"])


# --------------------------------------------------------------------------------------------
# Tower  [vision-API, DeepseekV4VisionTransformer.forward]: blocks in order, then the tower's
# `norm` (READING 8: applied after the last block; None skips it).  Starts from patch states
# [P, D] (the patch embedding is outside this path).
# --------------------------------------------------------------------------------------------
def tower_forward(x, layers, final_norm_w, grids, n_heads: int, rope_theta: float = 10000.0,
                  eps: float = 1e-6) -> np.ndarray:
    x = _f64(x)
    hd = x.shape[1] // n_heads
    cos, sin = packed_cos_sin(grids, hd // 2, rope_theta)
    for layer in layers:
        x = block_forward(x, layer, cos, sin, grids, n_heads, eps)
    if final_norm_w is not None:
        x = rmsnorm(x, final_norm_w, eps)
    return x


# --------------------------------------------------------------------------------------------
# Aligner  [vision-API, DeepseekV4VisionAligner]: spatially downsample each image's patch grid
# by downsample_ratio in both directions and project to the LLM width.
# READING 9: the grid is zero-padded at the bottom/right to a multiple of r; merged token
# (i, j) is the concatenation, over a (outer) and b (inner) in [0, r), of the patch vector at
# grid position (r*i + a, r*j + b) -> channel (a*r + b)*D + c; tokens are row-major over (i, j);
# the projection is one bias-free linear r*r*D -> E.
# --------------------------------------------------------------------------------------------
def patch_embed(patches, w_proj, bias=None) -> np.ndarray:
    """[vision-API, DeepseekV4VisionPatchEmbed]: a linear embedding of flattened RGB patches,
    [patches, 3, patch_h, patch_w] -> [patches, vision_dim], through the module's `proj`.
    READING 13: each patch is flattened in its own (channel, row, column) order, i.e. feature
    index c * patch_h * patch_w + i * patch_w + j, and `proj` is a Linear [D, 3 * patch_h *
    patch_w]; whether it has a bias is not stated, so the bias is optional (None = none)."""
    p = _f64(patches)
    flat = p.reshape(p.shape[0], -1)
    y = flat @ _f64(w_proj).T
    if bias is not None:
        y = y + _f64(bias)[None, :]
    return y


def aligner_merge(x, grids, r: int):
    """Returns the merged token matrix [T, r*r*D] and the token offsets [n_images + 1]."""
    x = _f64(x)
    d = x.shape[1]
    cu = cu_from_grids(grids)
    rows, cu_tok = [], [0]
    for (n_h, n_w), start in zip(grids, cu[:-1]):
        g_h, g_w = -(-n_h // r), -(-n_w // r)
        padded = np.zeros((g_h * r, g_w * r, d), dtype=np.float64)
        padded[:n_h, :n_w] = x[start:start + n_h * n_w].reshape(n_h, n_w, d)
        for i in range(g_h):
            for j in range(g_w):
                parts = [padded[r * i + a, r * j + b] for a in range(r) for b in range(r)]
                rows.append(np.concatenate(parts))
        cu_tok.append(cu_tok[-1] + g_h * g_w)
    return np.stack(rows), np.asarray(cu_tok, dtype=np.int64)


def aligner_forward(x, w_align, grids, r: int):
    merged, cu_tok = aligner_merge(x, grids, r)
    return merged @ _f64(w_align).T, cu_tok


def layer_norm(x, weight, bias, eps: float = 1e-6) -> np.ndarray:
    """LayerNorm over the last axis: (x - mean) / sqrt(var + eps) * weight + bias, population
    variance.  Used by the PatchMerger projector (see patch_merger)."""
    x = _f64(x)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * _f64(weight) + _f64(bias)


def gelu(z) -> np.ndarray:
    """Exact GELU, z * Phi(z) = z (1 + erf(z / sqrt 2)) / 2."""
    z = _f64(z)
    return 0.5 * z * (1.0 + np.vectorize(math.erf)(z / math.sqrt(2.0)))


def patch_merger_params(d: int, r: int, e: int) -> int:
    """Parameter count of the PatchMerger structure below: LayerNorm(d) weight and bias, Linear
    r^2 d -> r^2 d with bias, Linear r^2 d -> e with bias."""
    h = r * r * d
    return 2 * d + (h * h + h) + (h * e + e)


def patch_merger(x, grids, r: int, ln_w, ln_b, w1, b1, w2, b2, eps: float = 1e-6) -> np.ndarray:
    """The trained projector of [NVFP4 model card] ("merges each 2x2 group of patches and maps
    the resulting 4608-dimensional representation into the 4096-dimensional token space", 40,119,040
    parameters).  READING 14: the parameter count fixes a LayerNorm over each patch's d features,
    then Linear r^2 d -> r^2 d (+ bias), then Linear r^2 d -> e (+ bias) (patch_merger_params);
    the activation between the Linears is unstated and read as the exact GELU; the windows are
    merged exactly as aligner_merge (READING 9), a padding slot being a zero vector after the
    norm."""
    xn = layer_norm(x, ln_w, ln_b, eps)
    merged, cu_tok = aligner_merge(xn, grids, r)
    h = gelu(merged @ _f64(w1).T + _f64(b1)[None, :])
    return h @ _f64(w2).T + _f64(b2)[None, :], cu_tok


# --------------------------------------------------------------------------------------------
# Image-token bridge: [model-API, DeepseekV4Model] (sentinel parameters image_start, image_end,
# image_newline, image_pad; merge_image_embeddings; apply_deepseek_v4_image_visibility).
# READING 15: the integer codes of the pseudo-token types are not printed; -1 = text is stated.
# Taken: 0 = an image feature position, 1 = image_start, 2 = image_end, 3 = image_newline,
# 4 = image_pad.  The N-layout of one image of g_h x g_w aligner tokens is image_start, then
# each token row followed by image_newline, then image_end.  image_pad never appears in that
# layout; a caller may place it (e.g. to fill a bucket) and the merge gives it its sentinel.
# --------------------------------------------------------------------------------------------
TOK_TEXT, TOK_IMAGE, TOK_START, TOK_END, TOK_NEWLINE, TOK_PAD = -1, 0, 1, 2, 3, 4
SENTINEL_ORDER = (TOK_START, TOK_END, TOK_NEWLINE, TOK_PAD)  # rows of the sentinel matrix


def image_layout(n_h: int, n_w: int, r: int) -> np.ndarray:
    """Pseudo-token types of one image of an n_h x n_w patch grid (READING 15): the aligner gives
    ceil(n_h / r) rows of ceil(n_w / r) tokens (READING 9); each row is closed by a newline and
    the whole image is enclosed by start and end."""
    g_h, g_w = -(-n_h // r), -(-n_w // r)
    types = [TOK_START]
    for _ in range(g_h):
        types.extend([TOK_IMAGE] * g_w)
        types.append(TOK_NEWLINE)
    types.append(TOK_END)
    return np.asarray(types, dtype=np.int32)


def merge_image_embeddings(embeds, types, image_tokens, sentinels, tokens_per_image):
    """[model-API, DeepseekV4Model.merge_image_embeddings]: every pseudo-token row of the text
    embeddings is replaced; text rows (-1) are kept.

    embeds: [batch, seq, E]; types: [batch, seq]; image_tokens: [T, E], the aligner output of
    all images in packing order; sentinels: [4, E] in SENTINEL_ORDER; tokens_per_image: aligner
    tokens of each image in packing order.
    READING 16: the spans (image_spans, per sequence) taken in batch-major order are the images
    in packing order; the j-th span's feature positions take image j's tokens in order, and it
    must hold exactly that many.  Raises ValueError when the types do not fit the images."""
    out = np.array(embeds, copy=True)
    types = np.asarray(types)
    cu = np.concatenate([[0], np.cumsum(tokens_per_image)]).astype(np.int64)
    j = 0
    for b in range(types.shape[0]):
        for a, e in image_spans(types[b]):
            if j >= len(tokens_per_image):
                raise ValueError(f"more image spans than the {len(tokens_per_image)} images")
            k = cu[j]
            for p in range(a, e + 1):
                t = types[b, p]
                if t == TOK_IMAGE:
                    if k >= cu[j + 1]:
                        raise ValueError(f"span {j} holds more than {cu[j + 1] - cu[j]} features")
                    out[b, p] = image_tokens[k]
                    k += 1
                else:
                    out[b, p] = sentinels[SENTINEL_ORDER.index(t)]
            if k != cu[j + 1]:
                raise ValueError(f"span {j} holds {k - cu[j]} features, image {j} has {cu[j + 1] - cu[j]}")
            j += 1
    if j != len(tokens_per_image):
        raise ValueError(f"{j} image spans for {len(tokens_per_image)} images")
    return out


def image_spans(types_row):
    """Image spans of one sequence as inclusive (start, end) pairs.  READING 17: a span runs from
    an image_start to the next image_end and holds pseudo tokens only; a pseudo token outside
    such a pair, text inside one, an image_start inside an open span, a span left open at the
    end or an unknown type code is an error (ValueError)."""
    spans, open_at = [], None
    for p, t in enumerate(types_row):
        if t != TOK_TEXT and t != TOK_IMAGE and t not in SENTINEL_ORDER:
            raise ValueError(f"unknown pseudo-token type {t} at {p}")
        if t == TOK_TEXT:
            if open_at is not None:
                raise ValueError(f"text at {p} inside the span opened at {open_at}")
        elif t == TOK_START:
            if open_at is not None:
                raise ValueError(f"image_start at {p} inside the span opened at {open_at}")
            open_at = p
        elif t == TOK_END:
            if open_at is None:
                raise ValueError(f"image_end at {p} outside a span")
            spans.append((open_at, p))
            open_at = None
        elif open_at is None:
            raise ValueError(f"pseudo token {t} at {p} outside a span")
    if open_at is not None:
        raise ValueError(f"span opened at {open_at} is not closed")
    return spans


def image_visibility(mask, types):
    """[model-API, apply_deepseek_v4_image_visibility]: every pair of positions inside one image
    span becomes visible (additive 0); all other entries are kept.  mask: [batch, seq, seq]
    additive (the pages' [batch, 1, seq, seq] without the head axis); types: [batch, seq]."""
    out = np.array(mask, copy=True)
    for b in range(out.shape[0]):
        for a, e in image_spans(types[b]):
            out[b, a:e + 1, a:e + 1] = 0
    return out


def encode(inp, n_layers: int | None = None):
    """Whole path for one drawn input set (vision_transformer_encoder_dsv4v_b200.synth.Inputs):
    tower (first ``n_layers`` layers) then, if drawn, final norm and aligner.  Returns
    (tower_out [P, D], aligner_out [T, E] or None)."""
    wl = inp.wl
    layers = [{k: (t.values if hasattr(t, "values") else t) for k, t in layer.items()}
              for layer in inp.layers[:n_layers]]
    out = tower_forward(inp.x.values, layers, inp.final_norm_w, wl.grids, wl.n_heads,
                        wl.rope_theta, wl.eps)
    if inp.w_align is None:
        return out, None
    return out, aligner_forward(out, inp.w_align.values, wl.grids, wl.downsample_ratio)[0]

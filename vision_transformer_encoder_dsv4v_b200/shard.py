"""Image-parallel sharding of a packed batch across ranks.

Images never interact in the tower or the aligner, so a batch splits across GPUs by whole
images with no collective on the data path.  Each image costs about N (8 D^2 + 6 D F) + 4 N^2 D
flops per block (N = n_h * n_w); images are assigned longest-processing-time first to the
least-loaded rank, which keeps the ranks within one image of each other.
"""
from __future__ import annotations


def image_cost(n_h: int, n_w: int, vision_dim: int = 1024, mlp_hidden: int = 2816) -> float:
    n = n_h * n_w
    return n * (8.0 * vision_dim * vision_dim + 6.0 * vision_dim * mlp_hidden) + 4.0 * n * n * vision_dim


def shard_images(grids, world_size: int, vision_dim: int = 1024, mlp_hidden: int = 2816):
    """Returns, per rank, the indices of its images in ascending order (every image on exactly
    one rank)."""
    if world_size < 1:
        raise ValueError("world_size must be >= 1")
    order = sorted(range(len(grids)), key=lambda i: (-image_cost(*grids[i], vision_dim, mlp_hidden), i))
    loads = [0.0] * world_size
    parts = [[] for _ in range(world_size)]
    for i in order:
        r = min(range(world_size), key=lambda k: (loads[k], k))
        parts[r].append(i)
        loads[r] += image_cost(*grids[i], vision_dim, mlp_hidden)
    return [sorted(p) for p in parts]


def rank_batch(grids, world_size: int, rank: int, vision_dim: int = 1024, mlp_hidden: int = 2816):
    """The sub-batch (grids and the packed-row ranges of the full batch) that `rank` processes."""
    idx = shard_images(grids, world_size, vision_dim, mlp_hidden)[rank]
    cu = [0]
    for h, w in grids:
        cu.append(cu[-1] + h * w)
    return [grids[i] for i in idx], [(cu[i], cu[i + 1]) for i in idx]


def image_tokens(n_h: int, n_w: int, r: int) -> int:
    """Aligner tokens of one image: the grid padded to multiples of r, one token per window."""
    return -(-n_h // r) * -(-n_w // r)


def token_ranges(grids, r: int):
    """(start, end) of each image's tokens in the packed aligner output of the full batch."""
    out, t = [], 0
    for h, w in grids:
        n = image_tokens(h, w, r)
        out.append((t, t + n))
        t += n
    return out


def gather_tokens(local, grids, r: int, world_size: int, rank: int, group=None,
                  vision_dim: int = 1024, mlp_hidden: int = 2816):
    """All-gather(v) of the per-rank aligner outputs into the full batch's packed token order.

    `local` is this rank's [T_rank, E] output for the images `rank_batch` gave it (in that order);
    the result is the [T, E] output of the whole batch on every rank.  One collective: each rank
    pads its block to the largest rank's token count, `all_gather` moves the blocks (NCCL over
    NVLink on GPUs, gloo on CPU), and each image's rows are copied to their place in image order.
    """
    import torch
    import torch.distributed as dist

    parts = shard_images(grids, world_size, vision_dim, mlp_hidden)
    counts = [sum(image_tokens(*grids[i], r) for i in p) for p in parts]
    if local.shape[0] != counts[rank]:
        raise ValueError(f"rank {rank} holds {local.shape[0]} tokens, expected {counts[rank]}")
    width = local.shape[1]
    t_max = max(counts) if counts else 0
    padded = local.new_zeros((t_max, width))
    padded[: local.shape[0]] = local
    blocks = [torch.empty_like(padded) for _ in range(world_size)]
    dist.all_gather(blocks, padded, group=group)
    ranges = token_ranges(grids, r)
    total = ranges[-1][1] if ranges else 0
    out = local.new_empty((total, width))
    for k, p in enumerate(parts):
        o = 0
        for i in p:
            a, b = ranges[i]
            out[a:b] = blocks[k][o: o + (b - a)]
            o += b - a
    return out

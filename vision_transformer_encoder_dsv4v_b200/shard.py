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

"""The N > 1 path on CPU: image-parallel sharding over two gloo ranks.  Each rank runs the fp64
oracle on its images only; gathering the per-image results reproduces the single-process run
exactly (images never interact), and the max-over-ranks timing reduction behaves as the
benchmark uses it."""
import os

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import dsv4v_oracle as O
from vision_transformer_encoder_dsv4v_b200 import shard

GRIDS = [(3, 5), (2, 2), (4, 6), (1, 7), (5, 1), (3, 3)]


def test_token_ranges_follow_the_padded_windows():
    assert shard.image_tokens(3, 5, 2) == 6 and shard.image_tokens(4, 6, 2) == 6
    assert shard.image_tokens(1, 7, 2) == 4 and shard.image_tokens(28, 28, 2) == 196
    rng = shard.token_ranges([(3, 5), (2, 2), (27, 37)], 2)
    assert rng == [(0, 6), (6, 7), (7, 7 + 14 * 19)]


def test_shard_covers_every_image_once_and_balances():
    for world in (1, 2, 3, 4, 8):
        parts = shard.shard_images(GRIDS, world, 16, 32)
        flat = sorted(i for p in parts for i in p)
        assert flat == list(range(len(GRIDS)))
        loads = [sum(shard.image_cost(*GRIDS[i], 16, 32) for i in p) for p in parts]
        biggest = max(shard.image_cost(*g, 16, 32) for g in GRIDS)
        assert max(loads) - min(loads) <= biggest + 1e-9   # LPT: within one image
    grids5 = [(64, 64)] + [(8, 8)] * 15
    parts = shard.shard_images(grids5, 2)
    assert parts[0] == [0] or parts[1] == [0]               # the big image alone on one rank


def _worker(rank, world, port, out_q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(0)
        d, nh, f = 16, 2, 32
        cu = O.cu_from_grids(GRIDS)
        x = rng.normal(size=(int(cu[-1]), d))
        layer = dict(norm1_w=1 + 0.1 * rng.normal(size=d), wqkv=0.2 * rng.normal(size=(3 * d, d)),
                     wo=0.2 * rng.normal(size=(d, d)), norm2_w=1 + 0.1 * rng.normal(size=d),
                     w_gate=0.2 * rng.normal(size=(f, d)), w_up=0.2 * rng.normal(size=(f, d)),
                     w_down=0.2 * rng.normal(size=(d, f)))
        my_grids, rows = shard.rank_batch(GRIDS, world, rank, d, f)
        xs = np.concatenate([x[a:b] for a, b in rows]) if rows else np.zeros((0, d))
        y = O.tower_forward(xs, [layer], None, my_grids, nh) if my_grids else xs
        # gather everyone's (row range, result) and rebuild the packed output
        mine = [(a, b, y[o:o + (b - a)]) for (a, b), o in zip(rows, np.cumsum([0] + [b - a for a, b in rows])[:-1])]
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        full = np.zeros_like(x)
        for part in gathered:
            for a, b, blk in part:
                full[a:b] = blk
        ref = O.tower_forward(x, [layer], None, GRIDS, nh)
        # aligner on each rank's images, then the library's all-gather(v) of the tokens
        wa = 0.1 * rng.normal(size=(24, 4 * d))
        za = O.aligner_forward(y, wa, my_grids, 2)[0] if my_grids else np.zeros((0, 24))
        tok = shard.gather_tokens(torch.from_numpy(np.ascontiguousarray(za)), GRIDS, 2, world, rank,
                                  vision_dim=d, mlp_hidden=f)
        tok_ref = O.aligner_forward(ref, wa, GRIDS, 2)[0]
        tok_err = float(np.abs(tok.numpy() - tok_ref).max())
        # the benchmark's max-over-ranks reduction of per-rank times
        t = torch.tensor([float(rank + 1)])
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        out_q.put((rank, max(float(np.abs(full - ref).max()), tok_err), float(t.item())))
    finally:
        dist.destroy_process_group()


def test_two_rank_image_parallel_matches_single_process():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + (os.getpid() % 1000)
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, tmax in res:
        assert err <= 1e-12, (rank, err)   # each image's fp64 result does not depend on packing
        assert tmax == 2.0

"""Per-(batch, head) sharding of one problem over ranks (sharding.py), on the CPU.

The partition covers every slab exactly once in contiguous rank order, and two
gloo ranks that each compute their shard and all-gather reproduce a one-rank
computation exactly. The shard computation here is the fp64 oracle (standing in
for a GPU's kernels); the partition, views, padding and all-gather are the same
code the GPU path runs with NCCL.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_spherical_b200.configs import CONFIGS
from block_sparse_spherical_b200.sharding import ShardedBSA, shard_of


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("slabs,world", [(1, 1), (1, 2), (3, 2), (32, 8), (7, 4), (5, 8), (64, 3)])
def test_partition_covers_every_slab_once(slabs, world):
    owners = []
    prev_hi = 0
    for r in range(world):
        sh = shard_of(slabs, r, world)
        assert sh.lo == prev_hi and sh.lo <= sh.hi <= slabs and sh.slabs <= sh.chunk
        assert sh.chunk == -(-slabs // world)
        owners += [r] * sh.slabs
        prev_hi = sh.hi
    assert prev_hi == slabs and len(owners) == slabs
    assert owners == sorted(owners)


def test_partition_rejects_bad_requests():
    for args in ((0, 0, 1), (4, 2, 2), (4, -1, 2), (4, 0, 0)):
        with pytest.raises(ValueError):
            shard_of(*args)


def oracle_compute(cfg):
    """A shard's forward by the fp64 oracle: [1, s, N, d] float32 tensors -> [1, s, N, d]."""
    import oracle

    def run(q, k, v, g):
        outs = []
        for s in range(q.shape[1]):
            r = oracle.forward_slab(q[0, s].numpy(), k[0, s].numpy(), v[0, s].numpy(), g[0, s].numpy(),
                                    cfg.block_size, cfg.top_n, cfg.window_blocks)
            outs.append(torch.from_numpy(r["out"].astype(np.float32)))
        return torch.stack(outs)[None]
    return run


def full_inputs(cfg):
    from block_sparse_spherical_b200.synthetic import make_inputs
    q, k, v, g = make_inputs(cfg)
    return tuple(torch.from_numpy(np.ascontiguousarray(x)) for x in (q, k, v, g))


def _worker(rank, world, port, out_dir, heads):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        cfg = CONFIGS["tiny_nside8"].with_(heads=heads)
        q, k, v, g = full_inputs(cfg)
        layer = ShardedBSA(cfg.batch, cfg.heads, cfg.n_tokens, cfg.head_dim, cfg.block_size, cfg.top_n,
                           cfg.window_blocks, torch.float32, compute=oracle_compute(cfg))
        out = layer(q, k, v, g)
        local = layer(q, k, v, g, gather=False)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=out.numpy(), lo=layer.shard.lo, hi=layer.shard.hi,
                 local=np.zeros(0) if local is None else local.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("heads", [3, 1])
def test_two_gloo_ranks_reassemble_the_one_rank_output(tmp_path, heads):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path), heads), nprocs=world, join=True,
                       start_method="spawn")
    cfg = CONFIGS["tiny_nside8"].with_(heads=heads)
    q, k, v, g = full_inputs(cfg)
    whole = ShardedBSA(cfg.batch, cfg.heads, cfg.n_tokens, cfg.head_dim, cfg.block_size, cfg.top_n,
                       cfg.window_blocks, torch.float32, compute=oracle_compute(cfg))(q, k, v, g).numpy()
    r = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    for x in r:
        assert np.array_equal(x["out"], whole), "gathered output differs from the one-rank output"
    # each rank computed only its own slabs
    assert int(r[0]["lo"]) == 0 and int(r[1]["hi"]) == cfg.slabs and int(r[0]["hi"]) == int(r[1]["lo"])
    for x in r:
        lo, hi = int(x["lo"]), int(x["hi"])
        if hi > lo:
            assert np.array_equal(x["local"][0], whole.reshape(cfg.slabs, cfg.n_tokens, -1)[lo:hi])
        else:
            assert x["local"].size == 0

"""The multi-rank path of the benchmark on CPU: two gloo ranks (no GPU).

Each rank runs an independent replica of the workload (its own seed), the
ranks share nothing on the data path, and the reported step time is the max
over ranks. Here each rank runs the fp64 oracle on one small slab of its
replica (standing in for its GPU work), and the test checks the replica
seeds, the max-over-ranks reduction and the whole-job token count.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from block_sparse_spherical_b200.configs import CONFIGS
from block_sparse_spherical_b200.replicas import (barrier, job_head_rows_per_step, job_tokens_per_step,
                                                  max_over_ranks, replica_config)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from block_sparse_spherical_b200.synthetic import make_slab
        cfg = replica_config(CONFIGS["tiny_nside8"], rank)
        sl = make_slab(cfg, 0)
        barrier()
        res = oracle.forward_slab(sl.q, sl.k, sl.v, sl.gates, cfg.block_size, cfg.top_n, cfg.window_blocks)
        barrier()
        fake_ms = 10.0 + 5.0 * rank          # rank-dependent "device time"
        worst = max_over_ranks(fake_ms)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), out=res["out"], seed=cfg.seed, worst=worst,
                 tokens=job_tokens_per_step(cfg, world))
    finally:
        dist.destroy_process_group()


def test_two_gloo_replicas(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    r = [np.load(tmp_path / f"rank{i}.npz") for i in range(world)]
    assert int(r[0]["seed"]) == CONFIGS["tiny_nside8"].seed
    assert int(r[1]["seed"]) == CONFIGS["tiny_nside8"].seed + 1000
    assert not np.array_equal(r[0]["out"], r[1]["out"]), "replicas must run independent inputs"
    for x in r:
        assert float(x["worst"]) == 15.0          # max over ranks, seen by every rank
        assert int(x["tokens"]) == 2 * CONFIGS["tiny_nside8"].batch * CONFIGS["tiny_nside8"].n_tokens


def test_single_process_helpers_without_a_process_group():
    assert max_over_ranks(3.5) == 3.5
    barrier()
    cfg = CONFIGS["nside128"]
    assert replica_config(cfg, 0) is cfg
    assert job_tokens_per_step(cfg, 8) == 8 * 2 * 196608
    assert job_head_rows_per_step(cfg, 8) == 8 * 2 * 16 * 196608

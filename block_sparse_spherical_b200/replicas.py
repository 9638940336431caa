"""Multi-GPU plumbing of the benchmark: independent replicas, no data-path collective.

Every (batch, head) slab of BSA is an independent problem, so N ranks (one per
GPU) each run a full batch of their own ("weak" scaling). The only
communication is host-side bookkeeping through torch.distributed: a barrier
around the timed region and the max over ranks of the measured time. These
helpers are backend-agnostic (nccl on GPUs, gloo in the CPU tests).
"""
from __future__ import annotations

import os
from dataclasses import dataclass

import torch

from .configs import BSAConfig


@dataclass(frozen=True)
class RankInfo:
    rank: int
    world: int
    local_rank: int


def rank_info() -> RankInfo:
    """RANK / WORLD_SIZE / LOCAL_RANK as set by torchrun (single process: 0 / 1 / 0)."""
    return RankInfo(int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
                    int(os.environ.get("LOCAL_RANK", "0")))


def replica_config(cfg: BSAConfig, rank: int) -> BSAConfig:
    """The workload a rank runs: same shape, its own seed (rank 0 keeps the workload's)."""
    return cfg if rank == 0 else cfg.with_(seed=cfg.seed + 1000 * rank)


def max_over_ranks(value: float, device=None) -> float:
    """Max of a per-rank scalar (e.g. the timed region in ms) over all ranks."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None) -> None:
    if torch.distributed.is_available() and torch.distributed.is_initialized():
        if device is not None and torch.device(device).type == "cuda":
            torch.distributed.barrier(device_ids=[torch.device(device).index])
        else:
            torch.distributed.barrier()


def job_tokens_per_step(cfg: BSAConfig, world: int) -> int:
    """Tokens (batch x N; every head of a token counted once) processed by all ranks in one step
    (each rank runs a full batch)."""
    return world * cfg.batch * cfg.n_tokens


def job_head_rows_per_step(cfg: BSAConfig, world: int) -> int:
    """Query rows (batch x heads x N) processed by all ranks in one step."""
    return world * cfg.slabs * cfg.n_tokens

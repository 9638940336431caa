"""One BSA problem split over several GPUs by (batch, head) slab.

Every (batch, head) slab of BSA is an independent problem end to end: the
pooling, the compressed branch, the top-n choice and both fine branches of the
MOSAIC note's BSA section never mix slabs. So G ranks (one process per GPU)
each take a contiguous range of the B*H slabs and run the whole forward on it
with no communication; the only exchange is one all-gather that reassembles
the full output on every rank (NCCL over NVLink on GPUs, gloo in the CPU tests).

Partition: with c = ceil(B*H / G), rank r owns slabs [r*c, min((r+1)*c, B*H))
(the last ranks may own fewer, or none). In [B][H][N][d] memory a rank's slabs
are one contiguous span, so a shard is a view, and concatenating the ranks'
c-slab buffers in rank order restores slab order; the padding past B*H is cut.
A shard of s slabs runs as a problem with batch 1 and s heads (slabs only
differ in where they sit).

Two ways to reassemble (GPUs): gather="nccl" computes the shard into a local
buffer and runs one NCCL all-gather after it; gather="fused" keeps the full
output in symmetric memory on every rank and lets the fine-attention kernel's
epilogue store each finished row straight into every rank's buffer over NVLink
(bsa_forward_mirrored), so the exchange overlaps the computation tile by tile;
a symmetric-memory barrier then orders the stores before anyone reads. The
fused form uses plain peer stores (no multicast, no library kernel on peer
memory). It needs one GPU per rank, so it is not exercised on a single-GPU
machine; its per-GPU mechanics (the mirrored stores) are tested there with
local buffers.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist


@dataclass(frozen=True)
class Shard:
    rank: int
    world: int
    lo: int          # first slab of this rank
    hi: int          # one past its last slab
    chunk: int       # slabs per rank before trimming (c)

    @property
    def slabs(self) -> int:
        return self.hi - self.lo


def shard_of(total_slabs: int, rank: int, world: int) -> Shard:
    """The contiguous slab range of `rank` among `world` ranks."""
    if world < 1 or not 0 <= rank < world or total_slabs < 1:
        raise ValueError(f"bad partition request: slabs={total_slabs} rank={rank} world={world}")
    c = -(-total_slabs // world)
    lo = min(rank * c, total_slabs)
    return Shard(rank, world, lo, min(lo + c, total_slabs), c)


def _group_rank_world(group):
    if dist.is_available() and dist.is_initialized():
        return dist.get_rank(group), dist.get_world_size(group)
    return 0, 1


class ShardedBSA:
    """BSA forward over the slabs of one problem, split across the ranks of a process group.

    compute(q, k, v, gates) runs the forward of a shard ([1, s, N, d] tensors) and
    returns its output; by default it is the CUDA library (api.BSA). forward()
    takes the full [B, H, N, d] inputs on every rank, computes this rank's shard
    and, with gather=True, returns the full output on every rank; forward_local()
    takes and returns only this rank's shard.
    """

    def __init__(self, batch: int, heads: int, n_tokens: int, head_dim: int, block_size: int, top_n: int,
                 window_blocks: int = 1, dtype=torch.bfloat16, group=None, device=None, compute=None,
                 gather: str = "nccl"):
        self.shape = (batch, heads, n_tokens, head_dim)
        self.group = group
        rank, world = _group_rank_world(group)
        self.shard = shard_of(batch * heads, rank, world)
        self.dtype = dtype
        self.device = device
        if gather not in ("nccl", "fused"):
            raise ValueError(f"gather must be 'nccl' or 'fused', got {gather!r}")
        if gather == "fused" and (compute is not None or dtype != torch.bfloat16):
            raise ValueError("the fused gather runs the library's bf16 kernels")
        self.gather = gather
        self.layer = None
        if compute is None and self.shard.slabs > 0:
            from . import api
            self.layer = api.BSA(1, self.shard.slabs, n_tokens, head_dim, block_size, top_n, window_blocks, dtype,
                                 device=device if device is not None else "cuda")
            compute = self.layer
        self.compute = compute
        self._symm = None
        if gather == "fused":
            self._setup_symmetric(rank, world)

    def _setup_symmetric(self, rank, world):
        """Full output buffer in symmetric memory on every rank, and the views of the peers' buffers."""
        import torch.distributed._symmetric_memory as symm_mem
        b, h, n, d = self.shape
        dev = self.device if self.device is not None else torch.device("cuda", torch.cuda.current_device())
        self.full = symm_mem.empty(b * h, n, d, dtype=self.dtype, device=dev)
        group = self.group if self.group is not None else dist.group.WORLD
        self._symm = symm_mem.rendezvous(self.full, group)
        self.peers = [self._symm.get_buffer(r, (b * h, n, d), self.dtype) for r in range(world) if r != rank]

    def forward_local(self, q, k, v, gates):
        """This rank's shard: [1, s, N, d] inputs -> [1, s, N, d] output (None if it owns no slab)."""
        if self.shard.slabs == 0:
            return None
        return self.compute(q, k, v, gates)

    def forward(self, q, k, v, gates, gather: bool = True):
        b, h, n, d = self.shape
        for t in (q, k, v):
            if tuple(t.shape) != self.shape or not t.is_contiguous():
                raise ValueError(f"inputs must be contiguous {self.shape}")
        sh = self.shard
        view = lambda t, last: t.view(1, b * h, n, last)[:, sh.lo:sh.hi]
        if self.gather == "fused" and gather:
            return self._forward_fused(view(q, d), view(k, d), view(v, d), view(gates, 3))
        out_local = self.forward_local(view(q, d), view(k, d), view(v, d), view(gates, 3)) if sh.slabs else None
        if not gather:
            return out_local
        buf = torch.zeros((sh.chunk, n, d), dtype=q.dtype, device=q.device)
        if out_local is not None:
            buf[:sh.slabs].copy_(out_local.view(sh.slabs, n, d))
        if sh.world == 1:
            return buf[:b * h].view(b, h, n, d)
        full = torch.empty((sh.world * sh.chunk, n, d), dtype=q.dtype, device=q.device)
        dist.all_gather_into_tensor(full, buf, group=self.group)
        return full[:b * h].view(b, h, n, d)

    def _forward_fused(self, q, k, v, gates):
        from . import abi
        b, h, n, d = self.shape
        sh = self.shard
        if sh.slabs > 0:
            L = self.layer
            abi.bsa_forward_mirrored(L.cfg, q, k, v, gates, self.full[sh.lo:sh.hi],
                                     [p[sh.lo:sh.hi] for p in self.peers], L.sel_idx, L.workspace,
                                     L.workspace_bytes)
        self._symm.barrier()          # every rank's stores are complete and visible
        return self.full.view(b, h, n, d)

    __call__ = forward

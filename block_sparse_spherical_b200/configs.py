"""Named workloads for the BSA forward pass.

Each workload is a HEALPix NESTED token sequence: N = 12 * Nside**2 pixels
(MOSAIC note, "HEALPix spherical tessellation + NESTED index"), cut into
m = N / block_size contiguous blocks. With block_size = 4**L a block is exactly
the set of descendants of one pixel L levels coarser, because the children of
pixel p are 4p .. 4p+3 (same section).

This module holds sizes only; it performs none of the method's arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass, replace


@dataclass(frozen=True)
class BSAConfig:
    name: str
    nside: int
    batch: int
    heads: int
    head_dim: int
    block_size: int
    top_n: int
    window_blocks: int
    dtype: str  # "f32" or "bf16"
    seed: int
    tokens: int = 0  # explicit N for non-HEALPix test shapes; 0 means 12 * nside**2

    @property
    def n_tokens(self) -> int:
        return self.tokens if self.tokens else 12 * self.nside * self.nside

    @property
    def n_blocks(self) -> int:
        return self.n_tokens // self.block_size

    @property
    def slabs(self) -> int:
        return self.batch * self.heads

    @property
    def elt_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "BSAConfig":
        return replace(self, **kw)

    # ---- algorithmic work (what the method must do) ----
    def local_pairs_blocks(self) -> int:
        """Number of (query block, key block) pairs in the clamped local window."""
        m, w = self.n_blocks, self.window_blocks
        return sum(min(m - 1, i + w) - max(0, i - w) + 1 for i in range(m))

    def fine_flops(self) -> int:
        """QK^T + PV flops of the selection and local branches: 4*d per (query, key) pair."""
        pairs_blocks = self.n_blocks * min(self.top_n, self.n_blocks) + self.local_pairs_blocks()
        return 4 * self.head_dim * self.block_size * self.block_size * pairs_blocks * self.slabs

    def compressed_flops(self) -> int:
        """Block-level q̄k̄ᵀ and āv̄: 4*m*m*d per (batch, head)."""
        return 4 * self.n_blocks * self.n_blocks * self.head_dim * self.slabs

    def pool_bytes(self) -> int:
        """Bytes the pooling step must move: read q, k, v once, write three fp32 block means."""
        toks = self.slabs * self.n_tokens * self.head_dim
        return 3 * toks * self.elt_bytes + 3 * self.slabs * self.n_blocks * self.head_dim * 4

    def fused_min_bytes(self) -> int:
        """Minimum HBM bytes of the fused selection+local+combine kernel."""
        toks = self.slabs * self.n_tokens * self.head_dim
        return (4 * toks * self.elt_bytes                                  # q, k, v, out
                + self.slabs * self.n_tokens * 3 * 4                       # gates
                + self.slabs * self.n_blocks * self.head_dim * 4           # o_cg per block
                + self.slabs * self.n_blocks * self.top_n * 4)             # block indices

    def compress_min_bytes(self) -> int:
        """Minimum HBM bytes of compress+select: read q̄, k̄, v̄; write o_cg and indices."""
        blk = self.slabs * self.n_blocks * self.head_dim * 4
        return 4 * blk + self.slabs * self.n_blocks * self.top_n * 4


# The five workloads: sizes, dtypes and seeds as the method's evaluation grid
# names them (Nside 8 .. 256, i.e. about 7.3 to 0.23 degrees).
CONFIGS = {
    "tiny_nside8": BSAConfig("tiny_nside8", nside=8, batch=1, heads=2, head_dim=32,
                             block_size=16, top_n=4, window_blocks=1, dtype="f32", seed=0),
    "nside32": BSAConfig("nside32", nside=32, batch=1, heads=8, head_dim=64,
                         block_size=64, top_n=16, window_blocks=1, dtype="bf16", seed=1),
    "nside64": BSAConfig("nside64", nside=64, batch=4, heads=8, head_dim=64,
                         block_size=64, top_n=16, window_blocks=1, dtype="bf16", seed=2),
    "nside128": BSAConfig("nside128", nside=128, batch=2, heads=16, head_dim=64,
                          block_size=64, top_n=16, window_blocks=1, dtype="bf16", seed=3),
    "nside256": BSAConfig("nside256", nside=256, batch=1, heads=8, head_dim=64,
                          block_size=64, top_n=32, window_blocks=1, dtype="bf16", seed=4),
}

HEADLINE = "nside128"

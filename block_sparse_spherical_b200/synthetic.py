"""Seeded synthetic inputs shared by the CUDA path's tests/bench and the oracle.

Recipe (the workloads' description of the data): for every (batch, head) slab,
    q, k, v = 0.8 * u[block(t)] + 0.6 * eps[t]      u, eps ~ N(0, 1)
where u is one d-vector per block of `block_size` consecutive NESTED tokens
(drawn independently for q, k and v), eps is i.i.d. per element, and
    gates = sigmoid(N(0, 1))  of shape [N, 3], order (CG, FG, L).
bf16 workloads round q, k, v to bfloat16 (round to nearest, ties to even); the
same rounded values reach the GPU (as bf16 bits) and the oracle (widened).

Each slab draws from its own PCG64 stream, spawned from the workload seed, in
the fixed order u_q, u_k, u_v, eps_q, eps_k, eps_v, gate logits. Any slab can
therefore be regenerated alone, which keeps host memory bounded at Nside 256.

This module holds only the input recipe: none of the attention arithmetic.
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from .configs import BSAConfig


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (nearest, ties to even); return the 16-bit patterns."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    rounded = b + (np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1)))
    return (rounded >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Slab:
    """One (batch, head) slab. q/k/v hold exactly the values the kernels see."""
    q: np.ndarray      # [N, d] float32 (bf16-representable for bf16 workloads)
    k: np.ndarray
    v: np.ndarray
    gates: np.ndarray  # [N, 3] float32
    q_bits: np.ndarray | None = None  # [N, d] uint16 bf16 patterns (bf16 workloads)
    k_bits: np.ndarray | None = None
    v_bits: np.ndarray | None = None


def slab_streams(cfg: BSAConfig) -> list[np.random.SeedSequence]:
    return np.random.SeedSequence(cfg.seed).spawn(cfg.slabs)


def make_slab(cfg: BSAConfig, slab: int) -> Slab:
    """Generate slab number `slab` (= b * heads + h) of workload `cfg`."""
    ss = slab_streams(cfg)[slab]
    rng = np.random.Generator(np.random.PCG64(ss))
    n, d, bk, m = cfg.n_tokens, cfg.head_dim, cfg.block_size, cfg.n_blocks
    u = [rng.standard_normal((m, d), dtype=np.float32) for _ in range(3)]
    out = []
    for i in range(3):
        eps = rng.standard_normal((n, d), dtype=np.float32)
        x = np.float32(0.6) * eps
        x.reshape(m, bk, d)[...] += np.float32(0.8) * u[i][:, None, :]
        out.append(x)
    logits = rng.standard_normal((n, 3), dtype=np.float32)
    gates = (1.0 / (1.0 + np.exp(-logits.astype(np.float64)))).astype(np.float32)
    if cfg.dtype == "bf16":
        bits = [f32_to_bf16_bits(x) for x in out]
        vals = [bf16_bits_to_f32(b) for b in bits]
        return Slab(vals[0], vals[1], vals[2], gates, bits[0], bits[1], bits[2])
    return Slab(out[0], out[1], out[2], gates)


def make_inputs(cfg: BSAConfig):
    """Whole-workload inputs as host arrays in [B, H, N, d] / [B, H, N, 3] layout.

    Returns (q, k, v, gates): q/k/v are uint16 bf16 patterns for bf16 workloads
    and float32 for f32 workloads; gates are float32.
    """
    b, h, n, d = cfg.batch, cfg.heads, cfg.n_tokens, cfg.head_dim
    dt = np.uint16 if cfg.dtype == "bf16" else np.float32
    q = np.empty((b, h, n, d), dt)
    k = np.empty((b, h, n, d), dt)
    v = np.empty((b, h, n, d), dt)
    g = np.empty((b, h, n, 3), np.float32)
    for s in range(cfg.slabs):
        sl = make_slab(cfg, s)
        bi, hi = divmod(s, h)
        if cfg.dtype == "bf16":
            q[bi, hi], k[bi, hi], v[bi, hi] = sl.q_bits, sl.k_bits, sl.v_bits
        else:
            q[bi, hi], k[bi, hi], v[bi, hi] = sl.q, sl.k, sl.v
        g[bi, hi] = sl.gates
    return q, k, v, g


def to_float(cfg: BSAConfig, x: np.ndarray) -> np.ndarray:
    """Exact float32 values of an input array produced by make_inputs."""
    return bf16_bits_to_f32(x) if cfg.dtype == "bf16" else x

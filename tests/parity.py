"""Helpers shared by the GPU parity tests: device inputs from the seeded
generator, the oracle on sampled rows, and the acceptance rules.

Acceptance (the workloads' stated tolerances):
  * block indices: for every query block whose oracle gap z_(n) - z_(n+1)
    exceeds 1e-4 the GPU's index set equals the oracle's; for the others
    every GPU index is distinct, in [0, m) and has z_ij >= z_(n) - 1e-4;
  * outputs, compared with the oracle re-run on the GPU's indices:
    fp32 workloads max-abs <= 1e-4; bf16 workloads max-abs <= 2e-2 and
    mean-abs <= 2e-3;
  * pooled means and the block-level compressed output (fp32 on the GPU):
    max-abs <= 1e-4 for every workload.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from block_sparse_spherical_b200.synthetic import make_inputs, make_slab

GAP_TOL = 1e-4
FP32_TOL = 1e-4
BF16_MAX, BF16_MEAN = 2e-2, 2e-3


def device_inputs(cfg, device="cuda"):
    q, k, v, g = make_inputs(cfg)
    if cfg.dtype == "bf16":
        conv = lambda a: torch.from_numpy(a).view(torch.bfloat16).to(device)
    else:
        conv = lambda a: torch.from_numpy(a).to(device)
    return conv(q), conv(k), conv(v), torch.from_numpy(g).to(device)


def chunks_for(m: int, max_rows: int | None):
    """Contiguous query-block ranges to check: everything, or head/middle/tail."""
    if max_rows is None or m <= max_rows:
        return [(0, m)]
    c = max(1, max_rows // 3)
    mid = m // 2 - c // 2
    return [(0, c), (mid, mid + c), (m - c, m)]


def check_indices(gpu_idx, orc, n, what=""):
    """gpu_idx [R, n]; orc = oracle.compressed_rows(..., want_z=True) for the same rows."""
    gap, z, oidx = orc["gap"], orc["z"], orc["idx"]
    m = z.shape[1]
    exact = gap > GAP_TOL
    g_sorted = np.sort(gpu_idx, axis=1)
    o_sorted = np.sort(oidx, axis=1)
    bad = np.nonzero(exact & np.any(g_sorted != o_sorted, axis=1))[0]
    assert bad.size == 0, f"{what}: index set differs on {bad.size} rows with gap > {GAP_TOL} (first {bad[:5]})"
    assert np.all((gpu_idx >= 0) & (gpu_idx < m)), f"{what}: index out of range"
    assert np.all(np.diff(g_sorted, axis=1) != 0), f"{what}: repeated index"
    zn = np.take_along_axis(z, oidx[:, n - 1:n], axis=1)[:, 0]
    zg = np.take_along_axis(z, gpu_idx.astype(np.int64), axis=1)
    worst = float(np.min(zg - zn[:, None])) if zg.size else 0.0
    assert worst >= -GAP_TOL, f"{what}: a chosen block is {worst:.2e} below the n-th logit"
    return int(np.sum(~exact))


def check_output(got, want, dtype, what=""):
    err = np.abs(np.asarray(got, np.float64) - np.asarray(want, np.float64))
    mx, mean = float(err.max()), float(err.mean())
    if dtype == "f32":
        assert mx <= FP32_TOL, f"{what}: max abs {mx:.3e} > {FP32_TOL}"
    else:
        assert mx <= BF16_MAX and mean <= BF16_MEAN, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def to_np(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy()
    return t.cpu().numpy()


def check_slab(cfg, slab: int, gpu: dict, max_rows: int | None, q_scale: float = 1.0):
    """Compare one slab's GPU results with the oracle on sampled query blocks.

    gpu holds numpy arrays for this slab: qbar/kbar/vbar [m,d], o_cg [m,d],
    idx [m,n], out [N,d] (any may be missing). q_scale multiplies the seeded q
    (a power of two, so that the GPU's bf16 q scaled the same way is exact).
    Returns a summary dict.
    """
    s = make_slab(cfg, slab)
    bk, n, w = cfg.block_size, cfg.top_n, cfg.window_blocks
    q, k, v, g = (x.astype(np.float64) for x in (s.q, s.k, s.v, s.gates))
    q = q * q_scale
    qb, kb, vb = (oracle.pool(x, bk) for x in (q, k, v))
    summary = {"near_ties": 0, "out_max": 0.0, "out_mean": 0.0}
    for name, ob in (("qbar", qb), ("kbar", kb), ("vbar", vb)):
        if name in gpu:
            e = float(np.max(np.abs(gpu[name] - ob)))
            assert e <= FP32_TOL, f"{cfg.name} slab {slab} {name}: max abs {e:.3e}"
    m = cfg.n_blocks
    for r0, r1 in chunks_for(m, max_rows):
        orc = oracle.compressed_rows(qb, kb, vb, n, rows=(r0, r1), want_z=True)
        if "o_cg" in gpu:
            e = float(np.max(np.abs(gpu["o_cg"][r0:r1] - orc["o_cg"])))
            assert e <= FP32_TOL, f"{cfg.name} slab {slab} o_cg rows {r0}:{r1}: max abs {e:.3e}"
        if "idx" in gpu:
            summary["near_ties"] += check_indices(gpu["idx"][r0:r1], orc, n, f"{cfg.name} slab {slab}")
        if "out" in gpu:
            ocg = np.zeros((m, cfg.head_dim))
            ocg[r0:r1] = orc["o_cg"]
            f = oracle.fine_rows(q, k, v, g, ocg, gpu["idx"], bk, n, w, qblocks=(r0, r1))
            mx, mean = check_output(gpu["out"][r0 * bk:r1 * bk], f["out"], cfg.dtype,
                                    f"{cfg.name} slab {slab} out blocks {r0}:{r1}")
            summary["out_max"] = max(summary["out_max"], mx)
            summary["out_mean"] = max(summary["out_mean"], mean)
    return summary

"""numpy front end of the fp64 BSA oracle (bsa_oracle.c).

TEST INFRASTRUCTURE ONLY: imported by tests/, the package smoke check and the
benchmark's CPU-baseline leg; never by the product path. It shares no code
with the CUDA library and imports nothing from it.

Every function works on ONE (batch, head) slab: q, k, v are [N, d], gates
[N, 3]; inputs are converted to float64 (bf16 values widen exactly).
backward_slab gives the training gradients of the same forward.
"""
from __future__ import annotations

import ctypes
import math

import numpy as np

from . import build as _build

_lib = None

_dp = np.ctypeslib.ndpointer(dtype=np.float64, flags="C_CONTIGUOUS")
_ip = np.ctypeslib.ndpointer(dtype=np.int32, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64
_nullable_d = ctypes.c_void_p


def load(path: str | None = None):
    """Load (building first if needed) the oracle shared library."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    lib_path = path or _build.build()
    lib = ctypes.CDLL(lib_path)
    lib.oracle_pool.argtypes = [_i64, _i64, _i64, _dp, _dp]
    lib.oracle_compressed_rows.argtypes = [_i64, _i64, _i64, ctypes.c_double, _dp, _dp, _dp,
                                           _i64, _i64, _dp, _ip, _dp, _nullable_d]
    lib.oracle_fine_rows.argtypes = [_i64, _i64, _i64, _i64, _i64, ctypes.c_double,
                                     _dp, _dp, _dp, _dp, _dp, _ip, _i64, _i64,
                                     _dp, _nullable_d, _nullable_d]
    lib.oracle_forward_slab.argtypes = [_i64, _i64, _i64, _i64, _i64, ctypes.c_double,
                                        _dp, _dp, _dp, _dp, _nullable_d,
                                        _dp, _nullable_d, _nullable_d, _nullable_d,
                                        _nullable_d, _nullable_d, _nullable_d]
    lib.oracle_backward_slab.argtypes = [_i64, _i64, _i64, _i64, _i64, ctypes.c_double,
                                         _dp, _dp, _dp, _dp, _ip, _dp, _dp, _dp, _dp, _dp]
    lib.oracle_healpix_center.argtypes = [_i64, _i64, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_double)]
    lib.oracle_healpix_center.restype = None
    lib.oracle_latlon_plan.argtypes = [_i64, _i64, _i64, _ip, _dp]
    lib.oracle_interp.argtypes = [_i64, _i64, _i64, _i64, ctypes.c_double, _ip, _dp, _dp, _dp, _dp, _dp]
    for f in ("oracle_pool", "oracle_compressed_rows", "oracle_fine_rows", "oracle_forward_slab",
              "oracle_backward_slab", "oracle_latlon_plan", "oracle_interp"):
        getattr(lib, f).restype = ctypes.c_int
    if path is None:
        _lib = lib
    return lib


def load_native():
    """The oracle built with -O3 -march=native on this host (same results; for CPU timings)."""
    return load(_build.build_native())


def _f64(x) -> np.ndarray:
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def default_scale(d: int) -> float:
    return 1.0 / math.sqrt(d)


def pool(x, block: int, lib=None) -> np.ndarray:
    """Block means of x [N, d] over contiguous blocks of `block` tokens -> [m, d]."""
    lib = lib or load()
    x = _f64(x)
    n, d = x.shape
    out = np.empty((n // block, d), np.float64)
    if lib.oracle_pool(n, d, block, x, out) != 0:
        raise ValueError("oracle_pool: bad arguments")
    return out


def compressed_rows(qbar, kbar, vbar, n: int, scale: float | None = None, rows=None,
                    want_z: bool = False, lib=None):
    """Compressed branch + top-n for query blocks rows=(r0, r1).

    Returns dict(o_cg [r,d], idx [r,n] int32, gap [r], z [r,m] if want_z).
    """
    lib = lib or load()
    qbar, kbar, vbar = _f64(qbar), _f64(kbar), _f64(vbar)
    m, d = qbar.shape
    r0, r1 = rows if rows is not None else (0, m)
    scale = default_scale(d) if scale is None else scale
    r = r1 - r0
    o_cg = np.empty((r, d), np.float64)
    idx = np.empty((r, n), np.int32)
    gap = np.empty((r,), np.float64)
    z = np.empty((r, m), np.float64) if want_z else None
    rc = lib.oracle_compressed_rows(m, d, n, scale, qbar, kbar, vbar, r0, r1, o_cg, idx, gap, _ptr(z))
    if rc != 0:
        raise ValueError("oracle_compressed_rows: bad arguments")
    res = {"o_cg": o_cg, "idx": idx, "gap": gap}
    if want_z:
        res["z"] = z
    return res


def fine_rows(q, k, v, gates, o_cg, idx, block: int, n: int, w: int, scale: float | None = None,
              qblocks=None, want_branches: bool = False, lib=None):
    """Selection + local branches and gated combine for query blocks qblocks=(b0, b1).

    o_cg is the full [m, d] block-level compressed output, idx the full [m, n]
    index table. Returns dict(out [(b1-b0)*block, d], o_fg, o_l if asked).
    """
    lib = lib or load()
    q, k, v, gates, o_cg = _f64(q), _f64(k), _f64(v), _f64(gates), _f64(o_cg)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    ntok, d = q.shape
    m = ntok // block
    b0, b1 = qblocks if qblocks is not None else (0, m)
    scale = default_scale(d) if scale is None else scale
    rows = (b1 - b0) * block
    out = np.empty((rows, d), np.float64)
    ofg = np.empty((rows, d), np.float64) if want_branches else None
    ol = np.empty((rows, d), np.float64) if want_branches else None
    rc = lib.oracle_fine_rows(ntok, d, block, n, w, scale, q, k, v, gates, o_cg, idx, b0, b1,
                              out, _ptr(ofg), _ptr(ol))
    if rc != 0:
        raise ValueError("oracle_fine_rows: bad arguments")
    res = {"out": out}
    if want_branches:
        res["o_fg"], res["o_l"] = ofg, ol
    return res


def forward_slab(q, k, v, gates, block: int, n: int, w: int, scale: float | None = None,
                 forced_idx=None, lib=None):
    """Whole BSA forward of one slab. Returns dict(out, qbar, kbar, vbar, o_cg, idx, gap)."""
    lib = lib or load()
    q, k, v, gates = _f64(q), _f64(k), _f64(v), _f64(gates)
    ntok, d = q.shape
    m = ntok // block
    scale = default_scale(d) if scale is None else scale
    out = np.empty((ntok, d), np.float64)
    qb, kb, vb, ocg = (np.empty((m, d), np.float64) for _ in range(4))
    idx = np.empty((m, n), np.int32)
    gap = np.empty((m,), np.float64)
    fi = None if forced_idx is None else np.ascontiguousarray(forced_idx, dtype=np.int32)
    rc = lib.oracle_forward_slab(ntok, d, block, n, w, scale, q, k, v, gates, _ptr(fi), out,
                                 _ptr(qb), _ptr(kb), _ptr(vb), _ptr(ocg), _ptr(idx), _ptr(gap))
    if rc != 0:
        raise ValueError("oracle_forward_slab: bad arguments")
    return {"out": out, "qbar": qb, "kbar": kb, "vbar": vb, "o_cg": ocg, "idx": idx, "gap": gap}


def backward_slab(q, k, v, gates, idx, dout, block: int, n: int, w: int, scale: float | None = None,
                  lib=None):
    """Gradients of one slab's forward with the selection idx [m, n] held fixed.

    dout is dL/dout [N, d]. Returns dict(dq, dk, dv [N, d], dgates [N, 3]).
    """
    lib = lib or load()
    q, k, v, gates, dout = _f64(q), _f64(k), _f64(v), _f64(gates), _f64(dout)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    ntok, d = q.shape
    scale = default_scale(d) if scale is None else scale
    dq, dk, dv = (np.empty((ntok, d), np.float64) for _ in range(3))
    dg = np.empty((ntok, 3), np.float64)
    rc = lib.oracle_backward_slab(ntok, d, block, n, w, scale, q, k, v, gates, idx, dout, dq, dk, dv, dg)
    if rc != 0:
        raise ValueError("oracle_backward_slab: bad arguments")
    return {"dq": dq, "dk": dk, "dv": dv, "dgates": dg}


def healpix_centers(nside: int, lib=None) -> np.ndarray:
    """(z, phi) of every NESTED pixel centre at nside -> [12 nside^2, 2]."""
    lib = lib or load()
    n = 12 * nside * nside
    out = np.empty((n, 2), np.float64)
    z, ph = ctypes.c_double(), ctypes.c_double()
    for p in range(n):
        lib.oracle_healpix_center(nside, p, ctypes.byref(z), ctypes.byref(ph))
        out[p] = (z.value, ph.value)
    return out


def latlon_plan(nside: int, nlat: int, nlon: int, lib=None):
    """4 x 4 lat-lon neighbourhood (source indices [npix, 16]) and relative positions [npix, 16, 3]."""
    lib = lib or load()
    n = 12 * nside * nside
    nbr = np.empty((n, 16), np.int32)
    rel = np.empty((n, 16, 3), np.float64)
    if lib.oracle_latlon_plan(nside, nlat, nlon, nbr, rel) != 0:
        raise ValueError("oracle_latlon_plan: bad arguments")
    return nbr, rel


def interp(nbr, rel, wq, ksrc, vsrc, scale: float | None = None, lib=None) -> np.ndarray:
    """Cross-attention interpolation: out [n_tgt, d] from neighbours nbr [n_tgt, K], positions
    rel [n_tgt, K, 3], query map wq [d, 3] and source keys/values [n_src, d]."""
    lib = lib or load()
    nbr = np.ascontiguousarray(nbr, np.int32)
    rel, wq, ksrc, vsrc = _f64(rel), _f64(wq), _f64(ksrc), _f64(vsrc)
    n_tgt, K = nbr.shape
    n_src, d = ksrc.shape
    scale = default_scale(d) if scale is None else scale
    out = np.empty((n_tgt, d), np.float64)
    if lib.oracle_interp(n_tgt, K, d, n_src, scale, nbr, rel, wq, ksrc, vsrc, out) != 0:
        raise ValueError("oracle_interp: bad arguments")
    return out


__all__ = ["load", "load_native", "backward_slab", "healpix_centers", "latlon_plan", "interp", "pool", "compressed_rows", "fine_rows", "forward_slab", "default_scale"]

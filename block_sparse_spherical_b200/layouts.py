"""Token layouts for BSA other than HEALPix NESTED (the note's lat-lon-block ablation).

BSA cuts the token sequence into contiguous blocks. In HEALPix NESTED order a
block is one parent pixel, a compact equal-area patch (MOSAIC note, HEALPix
section). The note's ablation "BSA but not HEALPix (lat-lon block)" takes the
blocks from a regular latitude-longitude grid instead. Two readings of it are
provided here, both as permutations of a row-major (latitude, longitude)
raster of nlat x nlon points:
  * raster strips: the raster itself, cut into consecutive runs of block_size
    points along latitude rows (the identity permutation);
  * lat-lon patches: rectangles of patch_lat x patch_lon grid points, each made
    contiguous (patches row-major over the grid, points row-major inside).
`perm` lists, for every position of the block-contiguous order, the raster index
it takes (dst[t] = src[perm[t]], the convention of bsa_permute_tokens); `inverse`
undoes it. This module builds index arrays only; no attention arithmetic.
"""
from __future__ import annotations

import numpy as np


def raster_strips(nlat: int, nlon: int) -> np.ndarray:
    """Identity: blocks are consecutive raster points (strips along latitude rows)."""
    return np.arange(nlat * nlon, dtype=np.int32)


def latlon_patches(nlat: int, nlon: int, patch_lat: int, patch_lon: int) -> np.ndarray:
    """Block-contiguous order of patch_lat x patch_lon lat-lon patches."""
    if nlat % patch_lat or nlon % patch_lon:
        raise ValueError("the grid must split into whole patches")
    lat = np.arange(nlat).reshape(nlat // patch_lat, patch_lat)
    lon = np.arange(nlon).reshape(nlon // patch_lon, patch_lon)
    # axes: (patch row, patch column, row in patch, column in patch)
    idx = lat[:, None, :, None] * nlon + lon[None, :, None, :]
    return idx.reshape(-1).astype(np.int32)


def inverse(perm: np.ndarray) -> np.ndarray:
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size, dtype=perm.dtype)
    return inv

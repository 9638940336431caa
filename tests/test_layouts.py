"""Lat-lon token layouts (layouts.py) and the permutation entry point's host checks (CPU only)."""
import ctypes

import numpy as np
import pytest

from block_sparse_spherical_b200 import abi, build, layouts


@pytest.mark.parametrize("nlat,nlon,pl,pw", [(96, 128, 8, 8), (12, 20, 4, 5), (8, 8, 8, 8), (16, 32, 1, 32)])
def test_latlon_patches_are_contiguous_rectangles(nlat, nlon, pl, pw):
    perm = layouts.latlon_patches(nlat, nlon, pl, pw)
    assert perm.dtype == np.int32 and np.array_equal(np.sort(perm), np.arange(nlat * nlon))
    blk = pl * pw
    for b in range(perm.size // blk):
        pts = perm[b * blk:(b + 1) * blk]
        rows, cols = pts // nlon, pts % nlon
        assert rows.max() - rows.min() == pl - 1 and cols.max() - cols.min() == pw - 1
        assert len(set(zip(rows.tolist(), cols.tolist()))) == blk
    inv = layouts.inverse(perm)
    assert np.array_equal(perm[inv], np.arange(perm.size)) and np.array_equal(inv[perm], np.arange(perm.size))


def test_raster_strips_and_bad_grid():
    assert np.array_equal(layouts.raster_strips(3, 5), np.arange(15))
    with pytest.raises(ValueError):
        layouts.latlon_patches(10, 10, 3, 5)


def test_permute_tokens_host_validation():
    build.build()
    L = abi.load()
    A = 4096
    assert L.bsa_permute_tokens(0, 10, 128, A, A, A + 4096, None, None) == 1          # no slab
    assert L.bsa_permute_tokens(1, 10, 130, A, A, A + 4096, None, None) == 1          # row not a multiple of 4
    assert L.bsa_permute_tokens(1, 10, 128, None, A, A + 4096, None, None) == 1       # no permutation
    assert L.bsa_permute_tokens(1, 10, 128, A, A, A, None, None) == 1                 # in place
    assert L.bsa_permute_tokens(1, 10, 128, A, A + 4, A + 4096, None, None) == 3      # 16-byte rows, misaligned
    assert L.bsa_permute_tokens(1, 10, 12, A, A + 2, A + 4096, None, None) == 3       # 4-byte rows, misaligned

"""The fp64 oracle against facts fixed by the MOSAIC note and by mathematics (CPU only)."""
import math
import os

import numpy as np
import pytest

import oracle
import oracle_pins as pins
from block_sparse_spherical_b200.configs import CONFIGS

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(scope="module")
def lib():
    return oracle.load()


@pytest.mark.parametrize("check", pins.ALL_CHECKS, ids=lambda f: f.__name__)
def test_pin(lib, check):
    check(lib)


def test_healpix_counts_and_printed_resolutions():
    """N = 12 Nside^2 and the note's printed resolutions (golden file)."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "healpix_resolutions.txt"))
            if l.strip() and not l.startswith("#")]
    assert len(rows) == 4
    for nside_s, res_s in rows:
        nside, printed = int(nside_s), float(res_s)
        n_pix = 12 * nside * nside
        # equal-area pixels: angular size sqrt(4 pi / N) radians
        deg = math.degrees(math.sqrt(4.0 * math.pi / n_pix))
        assert abs(deg - printed) < 0.006, (nside, deg, printed)
        cfg = [c for c in CONFIGS.values() if c.nside == nside]
        assert cfg and all(c.n_tokens == n_pix for c in cfg)


def test_config_block_counts_and_work():
    """m = 12 (Nside / sqrt(B))^2 and the algorithmic work figures of each workload."""
    for cfg in CONFIGS.values():
        sqrt_b = int(round(math.sqrt(cfg.block_size)))
        assert sqrt_b * sqrt_b == cfg.block_size
        assert cfg.n_blocks == 12 * (cfg.nside // sqrt_b) ** 2
        assert cfg.n_tokens % cfg.block_size == 0
        # clamped window of +-1 block: 3 blocks inside, 2 at each end
        assert cfg.local_pairs_blocks() == 3 * cfg.n_blocks - 2
    c = CONFIGS["nside128"]
    assert c.n_tokens == 196608 and c.n_blocks == 3072
    assert abs(c.fine_flops() / 1e9 - 1958.4) < 0.1
    assert abs(c.compressed_flops() / 1e9 - 77.3) < 0.1


def test_descendant_ranges_closed_form():
    """Descendants of pixel P after L levels are [4^L P, 4^L P + 4^L) (induction on 4p..4p+3)."""
    for nside, levels in ((8, 2), (16, 1), (16, 4)):
        anc = pins.nested_ancestors(nside, levels)
        for p in range(0, 12 * (nside >> levels) ** 2, 5):
            members = np.nonzero(anc == p)[0]
            assert members.min() == 4 ** levels * p and len(members) == 4 ** levels
            assert np.all(np.diff(members) == 1)


def test_tiny_workload_full_forward(lib):
    """The tiny workload (Nside 8, fp32) through the oracle vs the masked-dense restatement."""
    from block_sparse_spherical_b200.synthetic import make_slab
    cfg = CONFIGS["tiny_nside8"]
    for s in range(cfg.slabs):
        sl = make_slab(cfg, s)
        r = oracle.forward_slab(sl.q, sl.k, sl.v, sl.gates, cfg.block_size, cfg.top_n,
                                cfg.window_blocks, lib=lib)
        want, idx = pins.masked_dense_restatement(
            sl.q.astype(np.float64), sl.k.astype(np.float64), sl.v.astype(np.float64),
            sl.gates.astype(np.float64), cfg.block_size, cfg.top_n, cfg.window_blocks,
            1.0 / math.sqrt(cfg.head_dim))
        assert np.array_equal(r["idx"], idx)
        assert np.max(np.abs(r["out"] - want)) < 1e-12


def test_oracle_rejects_bad_arguments(lib):
    x = np.zeros((10, 4))
    with pytest.raises(ValueError):
        oracle.pool(x, 3, lib=lib)   # N % B != 0
    qb = np.zeros((4, 2))
    with pytest.raises(ValueError):
        oracle.compressed_rows(qb, qb, qb, n=5, lib=lib)   # n > m
    with pytest.raises(ValueError):
        oracle.fine_rows(np.zeros((8, 2)), np.zeros((8, 2)), np.zeros((8, 2)), np.zeros((8, 3)),
                         np.zeros((2, 2)), np.array([[2], [0]], np.int32), 4, 1, 1, lib=lib)  # idx >= m

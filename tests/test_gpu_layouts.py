"""BSA over latitude-longitude blocks (the note's "BSA but not HEALPix" ablation) on the GPU.

bsa_permute_tokens moves rows between a lat-lon raster and block-contiguous
order (checked bit for bit against numpy indexing); BSA over lat-lon patches
is the permutation, bsa_forward, and the inverse permutation, compared with
the fp64 oracle run on the same permuted tokens under the workload tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_spherical_b200 import abi, api, layouts
from block_sparse_spherical_b200.configs import CONFIGS
from block_sparse_spherical_b200.synthetic import make_slab

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()


def test_permute_tokens_bit_exact():
    rng = np.random.default_rng(5)
    slabs, n = 3, 96 * 128
    perm = layouts.latlon_patches(96, 128, 8, 8)
    for width, dt in ((64, np.uint16), (3, np.float32), (64, np.float32)):
        x = rng.integers(0, 2 ** 16, size=(slabs, n, width)).astype(dt) if dt == np.uint16 else \
            rng.standard_normal((slabs, n, width)).astype(dt)
        src = torch.from_numpy(x).cuda()
        dst = torch.empty_like(src)
        row_bytes = width * x.itemsize
        abi.bsa_permute_tokens(slabs, n, row_bytes, torch.from_numpy(perm).cuda(), src, dst)
        torch.cuda.synchronize()
        assert np.array_equal(dst.cpu().numpy(), x[:, perm]), f"rows of {row_bytes} bytes"


def test_permute_tokens_flags_bad_index():
    n = 64
    perm = np.arange(n, dtype=np.int32)
    perm[5] = n
    src = torch.zeros((1, n, 64), dtype=torch.bfloat16, device="cuda")
    dst = torch.ones_like(src)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    abi.bsa_permute_tokens(1, n, 128, torch.from_numpy(perm).cuda(), src, dst, status)
    assert abi.bsa_check_status(status) == 7
    assert torch.equal(dst[0, 5], torch.ones_like(dst[0, 5])) and float(dst[0, 4].abs().max()) == 0.0


@pytest.mark.parametrize("layout", ["patches_8x8", "raster_strips"])
def test_bsa_over_latlon_blocks(layout):
    """A 96 x 128 lat-lon grid (12,288 points, as many as Nside 32) in blocks of 64 points."""
    nlat, nlon = 96, 128
    cfg = CONFIGS["nside32"].with_(name="latlon_" + layout, tokens=nlat * nlon, seed=41)
    perm = layouts.latlon_patches(nlat, nlon, 8, 8) if layout == "patches_8x8" else layouts.raster_strips(nlat, nlon)
    inv = layouts.inverse(perm)
    q, k, v, g = parity.device_inputs(cfg)             # fields in raster order
    dperm, dinv = torch.from_numpy(perm).cuda(), torch.from_numpy(inv).cuda()
    S, n = cfg.slabs, cfg.n_tokens

    def move(x, p):
        y = torch.empty_like(x)
        abi.bsa_permute_tokens(S, n, x.shape[-1] * x.element_size(), p, x, y)
        return y

    bsa = api.BSA.from_config(cfg)
    out = move(bsa(move(q, dperm), move(k, dperm), move(v, dperm), move(g, dperm)), dinv)
    torch.cuda.synchronize()
    assert bsa.check_status() == 0
    for slab in (0, S - 1):
        b, h = divmod(slab, cfg.heads)
        s = make_slab(cfg, slab)
        xs = [x.astype(np.float64)[perm] for x in (s.q, s.k, s.v, s.gates)]
        ref = oracle.forward_slab(*xs, cfg.block_size, cfg.top_n, cfg.window_blocks,
                                  forced_idx=bsa.sel_idx[b, h].cpu().numpy())
        orc = oracle.compressed_rows(ref["qbar"], ref["kbar"], ref["vbar"], cfg.top_n, want_z=True)
        parity.check_indices(bsa.sel_idx[b, h].cpu().numpy(), orc, cfg.top_n, f"{layout} slab {slab}")
        parity.check_output(parity.to_np(out[b, h]), ref["out"][inv], cfg.dtype, f"{layout} slab {slab}")

"""Lat-lon -> HEALPix cross-attention interpolation on the GPU against the fp64 oracle (needs a B200).

The plan's neighbour indices must equal the oracle's (the one floating-point
decision, the grid row under a pixel centre, may differ only where the centre
sits within 1e-9 rows of a grid row: there either neighbourhood is correct);
relative positions within 1e-5 (float32). The attention is compared with the
oracle run on the GPU's plan: fp32 features max-abs <= 1e-4; bf16 features
max-abs <= 2e-2 and mean-abs <= 2e-3 (the workloads' bounds).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_spherical_b200 import abi, api

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()


def check_plan(nside, nlat, nlon, layer):
    nbr, rel = oracle.latlon_plan(nside, nlat, nlon)
    g_nbr, g_rel = layer.nbr.cpu().numpy(), layer.rel.cpu().numpy()
    diff = np.nonzero(np.any(g_nbr != nbr, axis=1))[0]
    if diff.size:
        c = oracle.healpix_centers(nside)[diff]
        u = (90 - np.degrees(np.arcsin(c[:, 0]))) / (180 / (nlat - 1))
        assert np.all(np.abs(u - np.round(u)) < 1e-9), f"neighbourhoods differ at pixels {diff[:5]}"
    same = np.setdiff1d(np.arange(len(nbr)), diff)
    assert np.max(np.abs(g_rel[same] - rel[same])) <= 1e-5
    return g_nbr, g_rel


@pytest.mark.parametrize("nside,nlat,nlon", [(32, 121, 240), (8, 25, 48), (64, 181, 360)])
def test_plan_matches_oracle(nside, nlat, nlon):
    check_plan(nside, nlat, nlon, api.LatLonToHealpix(nside, nlat, nlon))


@pytest.mark.parametrize("nside,nlat,nlon,d,dtype,batch", [
    (32, 121, 240, 64, torch.float32, 2),     # 1.5 degree source onto Nside 32
    (32, 121, 240, 64, torch.bfloat16, 3),    # odd batch: the next image's kappa is loaded ahead
    (16, 61, 120, 32, torch.float32, 1),
    (16, 61, 120, 128, torch.bfloat16, 1),
    (256, 721, 1440, 64, torch.bfloat16, 1),  # 0.25 degree source onto Nside 256 (786,432 pixels)
])
def test_interp_matches_oracle(nside, nlat, nlon, d, dtype, batch):
    rng = np.random.default_rng(nside * 7 + d)
    n_src = nlat * nlon
    ks = rng.standard_normal((batch, n_src, d), dtype=np.float32)
    vs = rng.standard_normal((batch, n_src, d), dtype=np.float32)
    wq = (rng.standard_normal((d, 3)) / math.sqrt(3)).astype(np.float32)
    kt, vt = torch.from_numpy(ks).cuda().to(dtype), torch.from_numpy(vs).cuda().to(dtype)
    layer = api.LatLonToHealpix(nside, nlat, nlon)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = layer(kt, vt, torch.from_numpy(wq).cuda(), status_word=status)
    torch.cuda.synchronize()
    assert abi.bsa_check_status(status) == 0
    nbr, rel = layer.nbr.cpu().numpy(), layer.rel.cpu().numpy().astype(np.float64)
    npix = 12 * nside * nside
    rows = np.arange(npix) if npix <= 12 * 64 * 64 else np.concatenate(
        [np.arange(4096), np.arange(npix // 2, npix // 2 + 4096), np.arange(npix - 4096, npix)])
    for b in range(batch):
        kb, vb = kt[b].float().cpu().numpy(), vt[b].float().cpu().numpy()
        want = oracle.interp(nbr[rows], rel[rows], wq, kb, vb)
        parity.check_output(parity.to_np(out[b])[rows], want, "f32" if dtype == torch.float32 else "bf16",
                            f"interp nside {nside} d {d} batch {b}")


def test_interp_rejects_bad_arguments():
    L = abi.load()
    A = 4096
    assert L.bsa_latlon_to_healpix(1, 10, 10, 48, 1, 0.0, A, A, A, A, A, A, A, 4096, None, None) == 2   # head_dim 48
    assert L.bsa_latlon_to_healpix(1, 10, 10, 64, 5, 0.0, A, A, A, A, A, A, A, 4096, None, None) == 1   # dtype
    assert L.bsa_latlon_to_healpix(1, 10, 10, 64, 1, 0.0, A, A, A, A, A, A, A, 16, None, None) == 6     # workspace
    assert L.bsa_latlon_healpix_plan(3, 10, 10, A, A, None) == 1                              # nside not 2^k

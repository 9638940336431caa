"""The fine-attention kernel's FMA-pipe exp2: its coefficients are the Remez fit, its error bound
holds (CPU), and on the GPU it meets that bound against exact 2^x and tracks the exp unit."""
import os
import re

import numpy as np
import pytest

from block_sparse_spherical_b200.exp2_fit import remez_exp2

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "block_sparse_spherical_b200",
                   "csrc", "attend_tc.cu")
BOUND = 7.6e-5


def kernel_coefficients():
    body = open(SRC).read()
    body = body[body.index("float2 exp2_poly2"):]
    body = body[:body.index("return make_float2")]
    body = body[body.index("float2 p ="):]               # the polynomial, after the range reduction
    vals = [float.fromhex(h) for h in re.findall(r"(0x1\.[0-9a-f]+p-?\d+)f, 0x", body)]
    return vals  # c3, c2 (first FFMA2), c1, c0


def test_kernel_constants_are_the_remez_fit():
    c, err = remez_exp2(3)
    assert err < BOUND
    c3, c2, c1, c0 = kernel_coefficients()
    assert [c0, c1, c2, c3] == [float(np.float32(v)) for v in c]


@pytest.mark.gpu
def test_exp2_poly_on_gpu():
    import torch
    from block_sparse_spherical_b200 import abi
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    x = np.concatenate([np.linspace(-30, 8, 2_000_001, dtype=np.float32),
                        np.array([-125, -124.5, -0.5, 0.5, 0, 1, -1, 7.999], np.float32)])
    xt = torch.from_numpy(x).cuda()
    yp, ye = torch.empty_like(xt), torch.empty_like(xt)
    L = abi.load()
    assert L.bsa_testing_exp2(xt.data_ptr(), yp.data_ptr(), x.size, 1, None) == 0
    assert L.bsa_testing_exp2(xt.data_ptr(), ye.data_ptr(), x.size, 0, None) == 0
    torch.cuda.synchronize()
    exact = np.exp2(x.astype(np.float64))
    rp = np.abs(yp.cpu().numpy() / exact - 1)
    assert rp.max() <= BOUND * 1.01, f"polynomial exp2 relative error {rp.max():.3e}"
    re_ = np.abs(ye.cpu().numpy() / exact - 1)
    assert np.max(np.abs(yp.cpu().numpy() - ye.cpu().numpy()) / exact) <= BOUND + re_.max()
    # below the clamp the result stays tiny and positive instead of underflowing to garbage
    lo = torch.tensor([-200.0, -1000.0, -126.0, float("-inf")], device="cuda")
    out = torch.empty_like(lo)
    assert L.bsa_testing_exp2(lo.data_ptr(), out.data_ptr(), 4, 1, None) == 0
    o = out.cpu().numpy()
    assert np.all(o >= 0) and np.all(o < 2.0 ** -124)

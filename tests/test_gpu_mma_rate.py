"""The tensor-pipe rates the fine-attention roofline is stated against, measured by the library's
tcgen05.mma microbenchmark hook (include/bsa_testing.h): an M = 64 tile drives half of the
datapath of an M = 128 tile, and one issuing thread cannot keep the pipe busy with 64 x 64 tiles."""
import pytest
import torch

from block_sparse_spherical_b200 import abi

pytestmark = pytest.mark.gpu

MMAS = 256   # per warp


def mac_per_clk(m, n, warps):
    cyc = torch.zeros(warps, dtype=torch.int64, device="cuda")
    abi.bsa_testing_mma_rate(m, n, warps, cyc)
    torch.cuda.synchronize()
    c = cyc.cpu().tolist()
    assert min(c) > 0, f"bounded wait expired: {c}"
    return m * n * 16 * MMAS * warps / max(c)


def test_m64_is_half_of_m128():
    r64 = max(mac_per_clk(64, n, 4) for n in (64, 128, 256))
    r128 = max(mac_per_clk(128, n, 4) for n in (128, 256))
    # nominal dense bf16: 8192 flop = 4096 multiply-adds per clock per SM
    assert 3500 < r128 <= 4200, r128
    assert 0.4 < r64 / r128 < 0.6, (r64, r128)


def test_one_thread_cannot_fill_the_pipe_with_small_tiles():
    one = mac_per_clk(64, 64, 1)
    four = mac_per_clk(64, 64, 4)
    assert one < 0.8 * four, (one, four)


def test_rejects_other_shapes():
    cyc = torch.zeros(4, dtype=torch.int64, device="cuda")
    with pytest.raises(abi.BsaError):
        abi.bsa_testing_mma_rate(32, 64, 4, cyc)
    with pytest.raises(abi.BsaError):
        abi.bsa_testing_mma_rate(64, 64, 3, cyc)

"""The tensor-core kernel's bounded waits, exercised without faulting the GPU.

A test hook withholds one value-tile copy, so the MMA thread's wait for it
cannot complete; after its bound (about 2 s) the kernel must record a
timeout in the status word and return, and the CUDA context must stay
usable: a normal call afterwards gives the usual result.
"""
import ctypes

import pytest
import torch

from block_sparse_spherical_b200 import abi, api
from block_sparse_spherical_b200.configs import CONFIGS

import parity

pytestmark = pytest.mark.gpu


def test_withheld_copy_times_out_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    cfg = CONFIGS["nside32"]
    q, k, v, g = parity.device_inputs(cfg)
    qb, kb, vb = api.pool(q, k, v, cfg.block_size)
    o_cg, idx = api.compress_select(qb, kb, vb, cfg.top_n, cfg.block_size)
    good = api.fine_attention(q, k, v, g, o_cg, idx, cfg.block_size, cfg.window_blocks)
    torch.cuda.synchronize()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    c = abi.make_config(cfg)
    rc = abi.load().bsa_testing_fine_attention_withhold(
        ctypes.byref(c), q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), o_cg.data_ptr(),
        idx.data_ptr(), out.data_ptr(), status.data_ptr(), 5, torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    assert abi.bsa_check_status(status) == 5          # BSA_ERR_TIMEOUT
    assert abi.bsa_check_status(status) == 0          # reset
    again = api.fine_attention(q, k, v, g, o_cg, idx, cfg.block_size, cfg.window_blocks, status_word=status)
    assert abi.bsa_check_status(status) == 0
    assert torch.equal(again, good)

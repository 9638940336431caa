"""The allocation-free forward entry point (bsa_forward_noalloc), on a GPU.

bsa_forward_noalloc exists for callers that cannot allocate device memory
when they run BSA (allocator hooks, host callbacks, plugins whose framework
owns all device memory): it keeps its intermediates in a fixed scratch array
owned by the library. This test calls it through the C ABI twice in a row and
compares each result with bsa_forward (caller workspace): within the parity
tolerances of the other GPU tests and, as its header promises, bit for bit;
and it checks that a problem too large for the scratch is refused. It lives in its own file, collected last, and builds
its own inputs, so it passes alone in a fresh process or after the rest.
"""
import ctypes

import pytest
import torch

from block_sparse_spherical_b200 import abi, api
from block_sparse_spherical_b200.configs import CONFIGS

import parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()


@pytest.mark.parametrize("name", ["tiny_nside8", "nside32", "nside64"])
def test_noalloc_matches_workspace_forward_twice(name):
    cfg = CONFIGS[name]
    q, k, v, g = parity.device_inputs(cfg)
    ref_bsa = api.BSA.from_config(cfg)
    ref = ref_bsa(q, k, v, g)
    torch.cuda.synchronize()
    assert ref_bsa.check_status() == 0
    c = abi.make_config(cfg)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for call in range(2):
        out = torch.full_like(q, float("nan"))
        idx = torch.full_like(ref_bsa.sel_idx, -1)
        abi.bsa_forward_noalloc(c, q, k, v, g, out, idx, status)
        torch.cuda.synchronize()
        assert abi.bsa_check_status(status) == 0, f"call {call}: device status word set"
        assert torch.equal(idx, ref_bsa.sel_idx), f"call {call}: selected blocks differ"
        parity.check_output(parity.to_np(out), parity.to_np(ref), cfg.dtype, f"{name} no-alloc call {call}")
        # the header promises the same result as bsa_forward bit for bit
        assert torch.equal(out, ref), f"call {call}: output differs from bsa_forward"


def test_noalloc_without_optional_outputs():
    cfg = CONFIGS["nside32"]
    q, k, v, g = parity.device_inputs(cfg)
    ref = api.BSA.from_config(cfg)(q, k, v, g)
    out = torch.empty_like(q)
    abi.bsa_forward_noalloc(abi.make_config(cfg), q, k, v, g, out, None, None)
    torch.cuda.synchronize()
    parity.check_output(parity.to_np(out), parity.to_np(ref), cfg.dtype, "no-alloc without sel_idx/status")
    assert torch.equal(out, ref)


def test_noalloc_refuses_problems_beyond_its_scratch():
    cfg = CONFIGS["nside128"]
    c = abi.make_config(cfg)
    assert abi.bsa_workspace_size(c) > 32 << 20
    A = 1 << 20   # never dereferenced: the size check fails first
    rc = abi.load().bsa_forward_noalloc(ctypes.byref(c), A, A, A, A, A, None, None, None)
    assert rc == 6   # BSA_ERR_WORKSPACE

"""The C-ABI library without a GPU: it loads, exports every declared symbol,
and rejects bad arguments on the host before any launch (CPU only)."""
import ctypes
import os
import re

import pytest

from block_sparse_spherical_b200 import abi, build
from block_sparse_spherical_b200.configs import CONFIGS

INCLUDE = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return abi.load()


def declared_functions(header=None):
    names = []
    for h in sorted(os.listdir(INCLUDE)):
        if h.endswith(".h") and (header is None or h == header):
            src = open(os.path.join(INCLUDE, h)).read()
            names += re.findall(r"BSA_API\s+[\w\s\*]+?\b(bsa_\w+)\s*\(", src)
    return names


def test_header_declares_the_binding_names():
    assert sorted(declared_functions("bsa.h")) == sorted(abi.EXPORTS)
    assert sorted(declared_functions("bsa_testing.h")) == sorted(abi.TESTING_EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code, name in abi.STATUS_NAMES.items():
        assert abi.bsa_status_string(code).startswith(name)
    assert "UNKNOWN" in abi.bsa_status_string(99)


def cfg_of(**over):
    c = abi.make_config(CONFIGS["nside32"])
    for k, v in over.items():
        setattr(c, k, v)
    return c


def ws_size(c):
    n = ctypes.c_size_t(0)
    return abi.load().bsa_workspace_size(ctypes.byref(c), ctypes.byref(n)), n.value


@pytest.mark.parametrize("over,code", [
    (dict(batch=0), 1), (dict(heads=-1), 1), (dict(n_tokens=0), 1), (dict(head_dim=0), 1),
    (dict(block_size=0), 1), (dict(n_tokens=12289), 1), (dict(top_n=0), 1), (dict(top_n=193), 1),
    (dict(window_blocks=-1), 1), (dict(dtype=7), 1), (dict(scale=-1.0), 1), (dict(scale=float("nan")), 1),
    (dict(scale=float("inf")), 1),
    (dict(head_dim=128), 2), (dict(block_size=32), 2), (dict(dtype=0, block_size=16, head_dim=64), 2),
    (dict(top_n=65), 2), (dict(batch=70000), 2),
])
def test_workspace_size_validation(lib, over, code):
    rc, _ = ws_size(cfg_of(**over))
    assert rc == code


def test_workspace_size_layout(lib):
    for cfg in CONFIGS.values():
        c = abi.make_config(cfg)
        rc, n = ws_size(c)
        assert rc == 0
        pooled = cfg.slabs * cfg.n_blocks * cfg.head_dim * 4
        idx = cfg.slabs * cfg.n_blocks * cfg.top_n * 4
        up = lambda x: (x + 255) // 256 * 256
        split = 0
        if cfg.head_dim == 64 and cfg.top_n in (16, 32):   # tensor-core compressed path: tf32 split images
            m = cfg.n_blocks
            row_tiles, key_tiles = (m + 127) // 128, (m + 63) // 64
            split = cfg.slabs * (row_tiles * 65536 + 2 * key_tiles * 32768)
        assert n == 256 + 4 * up(pooled) + up(idx) + up(split)


def test_null_and_misaligned_pointers_rejected_before_launch(lib):
    c = abi.make_config(CONFIGS["nside32"])
    L = abi.load()
    cp = ctypes.byref(c)
    A = 4096          # never dereferenced: validation fails first
    # null pointers
    assert L.bsa_pool(cp, None, A, A, A, A, A, None) == 1
    assert L.bsa_compress_select(cp, A, A, A, A, None, None) == 1
    assert L.bsa_fine_attention(cp, A, A, A, A, A, A, None, None, None) == 1
    assert L.bsa_forward(cp, A, A, A, None, A, None, A, 1 << 30, None) == 1
    assert L.bsa_check_status(None, None) == 1
    # misalignment
    assert L.bsa_pool(cp, A + 2, A, A, A, A, A, None) == 3
    assert L.bsa_compress_select(cp, A, A, A + 8, A, A, None) == 3
    assert L.bsa_fine_attention(cp, A, A, A, A, A, A, A, A + 2, None) == 3
    assert L.bsa_forward(cp, A, A, A, A, A, None, A + 16, 1 << 30, None) == 3
    # workspace missing / too small
    assert L.bsa_forward(cp, A, A, A, A, A, None, None, 1 << 30, None) == 6
    assert L.bsa_compress_select_ws(cp, A, A, A, A, A, None, 1 << 30, None) == 6
    _, need = ws_size(c)
    assert L.bsa_forward(cp, A, A, A, A, A, None, A, need - 1, None) == 6
    assert L.bsa_compress_select_ws(cp, A, A, A, A, A, A, need - 1, None) == 6
    assert L.bsa_compress_select_ws(cp, A, A, A, A, A, A + 16, need, None) == 3
    # bad config with good pointers
    bad = cfg_of(top_n=0)
    assert L.bsa_forward(ctypes.byref(bad), A, A, A, A, A, None, A, need, None) == 1
    assert L.bsa_pool(None, A, A, A, A, A, A, None) == 1


def test_bf16_shape_beyond_the_tensor_core_kernel_is_an_error(lib):
    """bf16 fine attention runs on the tensor-core kernel only: a bf16 problem that kernel cannot
    address (more than 2^31 - 1 token rows for its 32-bit TMA coordinates) is refused with
    BSA_ERR_UNSUPPORTED on the host, never sent to another kernel."""
    L = abi.load()
    A = 4096          # never dereferenced: validation fails first
    big = cfg_of(batch=1, heads=2, n_tokens=1 << 30)
    assert L.bsa_fine_attention(ctypes.byref(big), A, A, A, A, A, A, A, None, None) == 2
    assert L.bsa_forward(ctypes.byref(big), A, A, A, A, A, None, A, 1 << 62, None) == 2
    assert ws_size(big)[0] == 2
    # the same row count in fp32 is a valid problem for the CUDA-core kernels
    assert ws_size(cfg_of(batch=1, heads=2, n_tokens=1 << 30, dtype=0))[0] == 0


def test_python_binding_raises_on_error(lib):
    c = cfg_of(top_n=0)
    with pytest.raises(abi.BsaError) as e:
        abi.bsa_workspace_size(c)
    assert e.value.code == 1


def test_python_binding_refuses_host_tensors(lib):
    """Every buffer of the library is device memory: the binding refuses a host tensor before the
    library is called (no host pointer ever reaches a kernel)."""
    import torch
    c = cfg_of()
    t = torch.zeros(16, dtype=torch.float32)
    with pytest.raises(ValueError, match="CUDA tensors"):
        abi.bsa_pool(c, t, t, t, t, t, t, stream=0)
    with pytest.raises(ValueError, match="CUDA tensors"):
        abi.bsa_check_status(t)

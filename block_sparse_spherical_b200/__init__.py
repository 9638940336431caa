"""B200-native forward pass of MOSAIC's mesh-aligned block-sparse attention (BSA).

The compute lives in libbsa.so (hand-written sm_100a CUDA behind a C ABI,
include/bsa.h); `abi` is its ctypes binding and `api` the torch-tensor front
end. Importing the package does not load the library; the first call does,
and fails loudly if it has not been built.
"""
from .configs import BSAConfig, CONFIGS, HEADLINE  # noqa: F401

__all__ = ["BSAConfig", "CONFIGS", "HEADLINE"]

"""Thin ctypes binding of libbsa.so (declared in include/bsa.h).

Argument marshalling only: every function here passes device pointers,
sizes and the current CUDA stream straight to the C ABI of the same name.
All computation happens in the library's CUDA kernels; if the library is
missing this module raises instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libbsa.so")

BSA_OK = 0
BSA_F32, BSA_BF16 = 0, 1
STATUS_NAMES = {
    0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_UNSUPPORTED", 3: "BSA_ERR_ALIGNMENT",
    4: "BSA_ERR_CUDA", 5: "BSA_ERR_TIMEOUT", 6: "BSA_ERR_WORKSPACE", 7: "BSA_ERR_INDEX",
}
EXPORTS = ("bsa_pool", "bsa_compress_select", "bsa_compress_select_ws", "bsa_fine_attention",
           "bsa_workspace_size", "bsa_forward", "bsa_check_status", "bsa_status_string", "bsa_forward_noalloc",
           "bsa_forward_train", "bsa_backward_workspace_size", "bsa_backward", "bsa_permute_tokens",
           "bsa_latlon_healpix_plan", "bsa_latlon_workspace_size", "bsa_latlon_to_healpix", "bsa_forward_mirrored")
TESTING_EXPORTS = ("bsa_testing_fine_attention_withhold", "bsa_testing_exp2", "bsa_testing_mma_rate")


class BsaConfig(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("n_tokens", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32), ("top_n", ctypes.c_int32),
                ("window_blocks", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


class BsaError(RuntimeError):
    def __init__(self, func: str, code: int):
        self.code = code
        super().__init__(f"{func} returned {STATUS_NAMES.get(code, code)}")


_lib = None


def load() -> ctypes.CDLL:
    """Load libbsa.so once; raise loudly if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libbsa.so is not built ({LIB_PATH}); run python -m block_sparse_spherical_b200.build")
    lib = ctypes.CDLL(LIB_PATH)
    P, S, C = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(BsaConfig)
    sig = {
        "bsa_pool": [C, P, P, P, P, P, P, P],
        "bsa_compress_select": [C, P, P, P, P, P, P],
        "bsa_compress_select_ws": [C, P, P, P, P, P, P, S, P],
        "bsa_fine_attention": [C, P, P, P, P, P, P, P, P, P],
        "bsa_workspace_size": [C, ctypes.POINTER(ctypes.c_size_t)],
        "bsa_forward": [C, P, P, P, P, P, P, P, S, P],
        "bsa_check_status": [P, P],
        "bsa_status_string": [ctypes.c_int],
        "bsa_forward_noalloc": [C, P, P, P, P, P, P, P, P],
        "bsa_forward_train": [C, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
        "bsa_backward_workspace_size": [C, ctypes.POINTER(ctypes.c_size_t)],
        "bsa_backward": [C, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, P, S, P],
        "bsa_permute_tokens": [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P, P, P, P, P],
        "bsa_latlon_healpix_plan": [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, P, P, P],
        "bsa_forward_mirrored": [C, P, P, P, P, P, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32, P, P, S, P],
        "bsa_latlon_workspace_size": [ctypes.c_int64, ctypes.c_int64, ctypes.POINTER(ctypes.c_size_t)],
        "bsa_latlon_to_healpix": [ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32,
                                  ctypes.c_float, P, P, P, P, P, P, P, S, P, P],
        "bsa_testing_fine_attention_withhold": [C, P, P, P, P, P, P, P, P, ctypes.c_int64, P],
        "bsa_testing_exp2": [P, P, ctypes.c_int64, ctypes.c_int32, P],
        "bsa_testing_mma_rate": [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, P, P],
    }
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "bsa_status_string" else ctypes.c_int
    _lib = lib
    return lib


def make_config(cfg, scale: float = 0.0) -> BsaConfig:
    """BsaConfig from a configs.BSAConfig (or any object with the same fields)."""
    return BsaConfig(cfg.batch, cfg.heads, cfg.n_tokens, cfg.head_dim, cfg.block_size, cfg.top_n,
                     cfg.window_blocks, BSA_BF16 if cfg.dtype == "bf16" else BSA_F32, scale)


def _ptr(t) -> int | None:
    """Address of a device buffer: None, a raw address, or a CUDA tensor (a host tensor is refused:
    every buffer argument of the library is device memory)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("buffer arguments must be CUDA tensors (device memory), got a host tensor")
    return t.data_ptr()


def _stream(stream) -> int | None:
    if stream is not None:
        return stream if isinstance(stream, int) else stream.cuda_stream
    import torch
    return torch.cuda.current_stream().cuda_stream


def _check(name: str, rc: int) -> None:
    if rc != BSA_OK:
        raise BsaError(name, rc)


def bsa_pool(cfg: BsaConfig, q, k, v, qbar, kbar, vbar, stream=None) -> None:
    _check("bsa_pool", load().bsa_pool(ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(qbar),
                                        _ptr(kbar), _ptr(vbar), _stream(stream)))


def bsa_compress_select(cfg: BsaConfig, qbar, kbar, vbar, o_cg_block, sel_idx, stream=None) -> None:
    _check("bsa_compress_select", load().bsa_compress_select(
        ctypes.byref(cfg), _ptr(qbar), _ptr(kbar), _ptr(vbar), _ptr(o_cg_block), _ptr(sel_idx),
        _stream(stream)))


def bsa_compress_select_ws(cfg: BsaConfig, qbar, kbar, vbar, o_cg_block, sel_idx, workspace, workspace_bytes: int,
                           stream=None) -> None:
    _check("bsa_compress_select_ws", load().bsa_compress_select_ws(
        ctypes.byref(cfg), _ptr(qbar), _ptr(kbar), _ptr(vbar), _ptr(o_cg_block), _ptr(sel_idx),
        _ptr(workspace), workspace_bytes, _stream(stream)))


def bsa_fine_attention(cfg: BsaConfig, q, k, v, gates, o_cg_block, sel_idx, out, status_word=None,
                       stream=None) -> None:
    _check("bsa_fine_attention", load().bsa_fine_attention(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(o_cg_block), _ptr(sel_idx),
        _ptr(out), _ptr(status_word), _stream(stream)))


def bsa_workspace_size(cfg: BsaConfig) -> int:
    n = ctypes.c_size_t(0)
    _check("bsa_workspace_size", load().bsa_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def bsa_forward(cfg: BsaConfig, q, k, v, gates, out, sel_idx_out, workspace, workspace_bytes: int,
                stream=None) -> None:
    _check("bsa_forward", load().bsa_forward(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(out), _ptr(sel_idx_out),
        _ptr(workspace), workspace_bytes, _stream(stream)))


def bsa_forward_noalloc(cfg: BsaConfig, q, k, v, gates, out, sel_idx_out=None, status_word=None,
                        stream=None) -> None:
    """bsa_forward without a caller workspace: the library's fixed 32 MiB device scratch is used."""
    _check("bsa_forward_noalloc", load().bsa_forward_noalloc(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(out), _ptr(sel_idx_out),
        _ptr(status_word), _stream(stream)))


def bsa_forward_train(cfg: BsaConfig, q, k, v, gates, out, sel_idx, o_cg_block, lse_cg, o_fg, o_l, lse_fine,
                      workspace, workspace_bytes: int, stream=None) -> None:
    _check("bsa_forward_train", load().bsa_forward_train(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(out), _ptr(sel_idx), _ptr(o_cg_block),
        _ptr(lse_cg), _ptr(o_fg), _ptr(o_l), _ptr(lse_fine), _ptr(workspace), workspace_bytes, _stream(stream)))


def bsa_backward_workspace_size(cfg: BsaConfig) -> int:
    n = ctypes.c_size_t(0)
    _check("bsa_backward_workspace_size", load().bsa_backward_workspace_size(ctypes.byref(cfg), ctypes.byref(n)))
    return n.value


def bsa_backward(cfg: BsaConfig, q, k, v, gates, dout, sel_idx, o_cg_block, lse_cg, o_fg, o_l, lse_fine,
                 dq, dk, dv, dgates, workspace, workspace_bytes: int, stream=None) -> None:
    _check("bsa_backward", load().bsa_backward(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(dout), _ptr(sel_idx), _ptr(o_cg_block),
        _ptr(lse_cg), _ptr(o_fg), _ptr(o_l), _ptr(lse_fine), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgates),
        _ptr(workspace), workspace_bytes, _stream(stream)))


def bsa_permute_tokens(slabs: int, n_tokens: int, row_bytes: int, perm, src, dst, status_word=None,
                       stream=None) -> None:
    _check("bsa_permute_tokens", load().bsa_permute_tokens(slabs, n_tokens, row_bytes, _ptr(perm), _ptr(src),
                                                           _ptr(dst), _ptr(status_word), _stream(stream)))


def bsa_latlon_healpix_plan(nside: int, nlat: int, nlon: int, nbr, rel, stream=None) -> None:
    _check("bsa_latlon_healpix_plan", load().bsa_latlon_healpix_plan(nside, nlat, nlon, _ptr(nbr), _ptr(rel),
                                                                     _stream(stream)))


def bsa_latlon_workspace_size(batch: int, n_src: int) -> int:
    n = ctypes.c_size_t(0)
    _check("bsa_latlon_workspace_size", load().bsa_latlon_workspace_size(batch, n_src, ctypes.byref(n)))
    return n.value


def bsa_latlon_to_healpix(batch: int, n_tgt: int, n_src: int, head_dim: int, dtype: int, scale: float, nbr, rel,
                          wq, k_src, v_src, out, workspace, workspace_bytes: int, status_word=None,
                          stream=None) -> None:
    _check("bsa_latlon_to_healpix", load().bsa_latlon_to_healpix(
        batch, n_tgt, n_src, head_dim, dtype, scale, _ptr(nbr), _ptr(rel), _ptr(wq), _ptr(k_src), _ptr(v_src),
        _ptr(out), _ptr(workspace), workspace_bytes, _ptr(status_word), _stream(stream)))


def bsa_forward_mirrored(cfg: BsaConfig, q, k, v, gates, out, mirrors, sel_idx_out, workspace,
                         workspace_bytes: int, stream=None) -> None:
    arr = (ctypes.c_void_p * max(1, len(mirrors)))(*[_ptr(m) for m in mirrors])
    _check("bsa_forward_mirrored", load().bsa_forward_mirrored(
        ctypes.byref(cfg), _ptr(q), _ptr(k), _ptr(v), _ptr(gates), _ptr(out), arr, len(mirrors),
        _ptr(sel_idx_out), _ptr(workspace), workspace_bytes, _stream(stream)))


def bsa_testing_mma_rate(m: int, n: int, warps: int, cycles, stream=None) -> None:
    """Test hook: each of `warps` warps' cycles for 256 back-to-back m x n bf16 tcgen05.mma (K=16)."""
    _check("bsa_testing_mma_rate", load().bsa_testing_mma_rate(m, n, warps, _ptr(cycles), _stream(stream)))


def bsa_check_status(status_word, stream=None) -> int:
    """Return the status code (0 = BSA_OK) after syncing `stream`; the word is reset."""
    return load().bsa_check_status(_ptr(status_word), _stream(stream))


def bsa_status_string(code: int) -> str:
    return load().bsa_status_string(code).decode()

"""torch-tensor front end of the BSA C ABI.

PyTorch supplies device memory and the current stream; each call marshals
tensors into one C-ABI call (abi.py) and the kernels in libbsa.so do all the
work. Inputs must be contiguous CUDA tensors in the layouts of include/bsa.h.
"""
from __future__ import annotations

import torch

from . import abi


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return abi.BSA_BF16
    if t.dtype == torch.float32:
        return abi.BSA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _require(t: torch.Tensor, name: str, dtype=None, shape=None):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def config_for(q: torch.Tensor, block_size: int, top_n: int, window_blocks: int = 1,
               scale: float = 0.0) -> abi.BsaConfig:
    b, h, n, d = q.shape
    return abi.BsaConfig(b, h, n, d, block_size, top_n, window_blocks, _dtype_code(q), scale)


class BSA:
    """A BSA forward pass of fixed shape with its workspace held on the device.

    Calling the object runs pool -> compress/select -> fine attention on the
    current stream (three kernels) and returns `out` ([B, H, N, d], q's dtype).
    """

    def __init__(self, batch: int, heads: int, n_tokens: int, head_dim: int, block_size: int,
                 top_n: int, window_blocks: int = 1, dtype=torch.bfloat16, scale: float = 0.0,
                 device="cuda"):
        self.cfg = abi.BsaConfig(batch, heads, n_tokens, head_dim, block_size, top_n, window_blocks,
                                 abi.BSA_BF16 if dtype == torch.bfloat16 else abi.BSA_F32, scale)
        self.shape = (batch, heads, n_tokens, head_dim)
        self.dtype = dtype
        self.m = n_tokens // block_size
        self.workspace_bytes = abi.bsa_workspace_size(self.cfg)
        self.workspace = torch.zeros(self.workspace_bytes, dtype=torch.uint8, device=device)
        self.sel_idx = torch.empty((batch, heads, self.m, top_n), dtype=torch.int32, device=device)

    @classmethod
    def from_config(cls, cfg, device="cuda", scale: float = 0.0) -> "BSA":
        return cls(cfg.batch, cfg.heads, cfg.n_tokens, cfg.head_dim, cfg.block_size, cfg.top_n,
                   cfg.window_blocks, torch.bfloat16 if cfg.dtype == "bf16" else torch.float32, scale,
                   device)

    def __call__(self, q, k, v, gates, out=None) -> torch.Tensor:
        for name, t in (("q", q), ("k", k), ("v", v)):
            _require(t, name, self.dtype, self.shape)
        _require(gates, "gates", torch.float32, self.shape[:3] + (3,))
        if out is None:
            out = torch.empty_like(q)
        _require(out, "out", self.dtype, self.shape)
        abi.bsa_forward(self.cfg, q, k, v, gates, out, self.sel_idx, self.workspace, self.workspace_bytes)
        return out

    def check_status(self) -> int:
        """Synchronise and return the kernels' status code (0 = OK); resets it."""
        return abi.bsa_check_status(self.workspace)


class BSAStream:
    """BSA forwards over a sequence of batches held in pinned host memory, with the host-device
    copies overlapped with the computation.

    run(batches, outs) enqueues, for batch i: its inputs copied in on a copy stream into device
    buffer set i % 2, the forward (bsa_forward) on a compute stream, and its output copied back on
    a third stream into outs[i]; so batch i+1's inputs move in and batch i-1's output moves out
    while batch i computes. Events order the reuse of each buffer set (inputs: after the forward
    two batches back has read them; output: after the copy-out two batches back has read it).
    run returns once everything is enqueued; synchronize() waits for it. The host tensors must
    stay alive and unchanged until then. The device buffers (and the layer's workspace and index
    array) are marked as used by the streams that touch them, so that memory freed with this object
    is not handed out again while a copy or a forward on one of them is still pending.
    """

    def __init__(self, layer: BSA):
        self.layer = layer
        dev = layer.workspace.device
        b, h, n, d = layer.shape
        self.streams = [torch.cuda.Stream(dev) for _ in range(3)]   # copy in, compute, copy out
        self.bufs = [dict(q=torch.empty(layer.shape, dtype=layer.dtype, device=dev),
                          k=torch.empty(layer.shape, dtype=layer.dtype, device=dev),
                          v=torch.empty(layer.shape, dtype=layer.dtype, device=dev),
                          gates=torch.empty((b, h, n, 3), dtype=torch.float32, device=dev),
                          out=torch.empty(layer.shape, dtype=layer.dtype, device=dev)) for _ in range(2)]
        for buf in self.bufs:
            for t in buf.values():
                for st in self.streams:
                    t.record_stream(st)
        layer.workspace.record_stream(self.streams[1])
        layer.sel_idx.record_stream(self.streams[1])
        self.in_done = [torch.cuda.Event() for _ in range(2)]
        self.cmp_done = [torch.cuda.Event() for _ in range(2)]
        self.out_done = [torch.cuda.Event() for _ in range(2)]
        self._used = [False, False]

    def run(self, batches, outs) -> None:
        s_in, s_cmp, s_out = self.streams
        for i, ((q, k, v, gates), o) in enumerate(zip(batches, outs)):
            for name, t in (("q", q), ("k", k), ("v", v), ("gates", gates), ("out", o)):
                if t.is_cuda or not t.is_pinned():
                    raise ValueError(f"{name} of batch {i} must be a pinned host tensor")
            j = i % 2
            buf = self.bufs[j]
            with torch.cuda.stream(s_in):
                if self._used[j]:
                    s_in.wait_event(self.cmp_done[j])
                for name, t in (("q", q), ("k", k), ("v", v), ("gates", gates)):
                    buf[name].copy_(t, non_blocking=True)
                self.in_done[j].record(s_in)
            with torch.cuda.stream(s_cmp):
                s_cmp.wait_event(self.in_done[j])
                if self._used[j]:
                    s_cmp.wait_event(self.out_done[j])
                self.layer(buf["q"], buf["k"], buf["v"], buf["gates"], out=buf["out"])
                self.cmp_done[j].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(self.cmp_done[j])
                o.copy_(buf["out"], non_blocking=True)
                self.out_done[j].record(s_out)
            self._used[j] = True

    def synchronize(self) -> None:
        for st in self.streams:
            st.synchronize()


class BSATrain(BSA):
    """A BSA layer of fixed shape for training: forward() saves what backward() needs.

    forward(q, k, v, gates) -> out; backward(dout) -> (dq, dk, dv, dgates), with the
    selected blocks held fixed. bf16, block 64, head_dim 64. The saved tensors and
    both workspaces live on the device between the two calls.
    """

    def __init__(self, *args, **kw):
        super().__init__(*args, **kw)
        b, h, n, d = self.shape
        dev = self.workspace.device
        self.o_cg = torch.empty((b, h, self.m, d), dtype=torch.float32, device=dev)
        self.lse_cg = torch.empty((b, h, self.m), dtype=torch.float32, device=dev)
        self.o_fg = torch.empty(self.shape, dtype=self.dtype, device=dev)
        self.o_l = torch.empty(self.shape, dtype=self.dtype, device=dev)
        self.lse_fine = torch.empty((b, h, n, 2), dtype=torch.float32, device=dev)
        self.bwd_workspace_bytes = abi.bsa_backward_workspace_size(self.cfg)
        self.bwd_workspace = torch.zeros(self.bwd_workspace_bytes, dtype=torch.uint8, device=dev)
        self._saved = None

    def __call__(self, q, k, v, gates, out=None) -> torch.Tensor:
        return self.forward(q, k, v, gates, out)

    def forward(self, q, k, v, gates, out=None) -> torch.Tensor:
        for name, t in (("q", q), ("k", k), ("v", v)):
            _require(t, name, self.dtype, self.shape)
        _require(gates, "gates", torch.float32, self.shape[:3] + (3,))
        if out is None:
            out = torch.empty_like(q)
        _require(out, "out", self.dtype, self.shape)
        abi.bsa_forward_train(self.cfg, q, k, v, gates, out, self.sel_idx, self.o_cg, self.lse_cg, self.o_fg,
                              self.o_l, self.lse_fine, self.workspace, self.workspace_bytes)
        self._saved = (q, k, v, gates)
        return out

    def backward(self, dout, grads=None):
        """Gradients (dq, dk, dv, dgates) of the last forward() for dL/dout = dout."""
        if self._saved is None:
            raise RuntimeError("backward() needs a forward() first")
        q, k, v, gates = self._saved
        _require(dout, "dout", self.dtype, self.shape)
        if grads is None:
            grads = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(gates))
        dq, dk, dv, dg = grads
        abi.bsa_backward(self.cfg, q, k, v, gates, dout, self.sel_idx, self.o_cg, self.lse_cg, self.o_fg, self.o_l,
                         self.lse_fine, dq, dk, dv, dg, self.bwd_workspace, self.bwd_workspace_bytes)
        return dq, dk, dv, dg

    def check_backward_status(self) -> int:
        """Synchronise and return the backward kernels' status code (0 = OK); resets it."""
        return abi.bsa_check_status(self.bwd_workspace)


class LatLonToHealpix:
    """Cross-attention interpolation from a lat-lon grid to the HEALPix NESTED pixels at nside.

    The plan (16 neighbours and relative positions per pixel) is built once on the
    device; calling the object with k_src, v_src [B, nlat*nlon, d] (bf16 or fp32) and
    the query map wq [d, 3] (fp32) returns [B, 12*nside^2, d].
    """

    def __init__(self, nside: int, nlat: int, nlon: int, device="cuda"):
        self.nside, self.nlat, self.nlon = nside, nlat, nlon
        self.npix = 12 * nside * nside
        self.nbr = torch.empty((self.npix, 16), dtype=torch.int32, device=device)
        self.rel = torch.empty((self.npix, 16, 3), dtype=torch.float32, device=device)
        abi.bsa_latlon_healpix_plan(nside, nlat, nlon, self.nbr, self.rel)
        self._ws = None            # the keys' 3-float position-space images, sized on first use

    def __call__(self, k_src, v_src, wq, scale: float = 0.0, out=None, status_word=None):
        b, n_src, d = k_src.shape
        if n_src != self.nlat * self.nlon:
            raise ValueError(f"k_src must hold {self.nlat * self.nlon} grid points, got {n_src}")
        _require(k_src, "k_src")
        _require(v_src, "v_src", k_src.dtype, k_src.shape)
        _require(wq, "wq", torch.float32, (d, 3))
        if out is None:
            out = torch.empty((b, self.npix, d), dtype=k_src.dtype, device=k_src.device)
        _require(out, "out", k_src.dtype, (b, self.npix, d))
        need = abi.bsa_latlon_workspace_size(b, n_src)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(need, dtype=torch.uint8, device=k_src.device)
        abi.bsa_latlon_to_healpix(b, self.npix, n_src, d, _dtype_code(k_src), scale, self.nbr, self.rel, wq, k_src,
                                  v_src, out, self._ws, self._ws.numel(), status_word)
        return out


def forward(q, k, v, gates, block_size: int, top_n: int, window_blocks: int = 1, scale: float = 0.0,
            return_indices: bool = False):
    """One-shot BSA forward (allocates a workspace; use BSA for repeated calls)."""
    b, h, n, d = q.shape
    bsa = BSA(b, h, n, d, block_size, top_n, window_blocks, q.dtype, scale, q.device)
    out = bsa(q, k, v, gates)
    return (out, bsa.sel_idx) if return_indices else out


def pool(q, k, v, block_size: int):
    """Block means of q, k, v -> three float32 tensors [B, H, m, d]."""
    b, h, n, d = q.shape
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require(t, name, q.dtype, q.shape)
    cfg = config_for(q, block_size, 1, 0)
    outs = [torch.empty((b, h, n // block_size, d), dtype=torch.float32, device=q.device) for _ in range(3)]
    abi.bsa_pool(cfg, q, k, v, *outs)
    return tuple(outs)


def compress_select(qbar, kbar, vbar, top_n: int, block_size: int, dtype=torch.bfloat16,
                    scale: float = 0.0):
    """Compressed branch + top-n from pooled tensors -> (o_cg_block [B,H,m,d], sel_idx [B,H,m,n])."""
    b, h, m, d = qbar.shape
    for name, t in (("qbar", qbar), ("kbar", kbar), ("vbar", vbar)):
        _require(t, name, torch.float32, qbar.shape)
    cfg = abi.BsaConfig(b, h, m * block_size, d, block_size, top_n, 0,
                        abi.BSA_BF16 if dtype == torch.bfloat16 else abi.BSA_F32, scale)
    o_cg = torch.empty_like(qbar)
    idx = torch.empty((b, h, m, top_n), dtype=torch.int32, device=qbar.device)
    abi.bsa_compress_select(cfg, qbar, kbar, vbar, o_cg, idx)
    return o_cg, idx


def fine_attention(q, k, v, gates, o_cg_block, sel_idx, block_size: int, window_blocks: int = 1,
                   scale: float = 0.0, status_word=None, out=None):
    """Selection + local branches and gated combine from given o_cg_block and sel_idx."""
    b, h, n, d = q.shape
    top_n = sel_idx.shape[-1]
    for name, t in (("q", q), ("k", k), ("v", v)):
        _require(t, name, q.dtype, q.shape)
    _require(gates, "gates", torch.float32, (b, h, n, 3))
    _require(o_cg_block, "o_cg_block", torch.float32, (b, h, n // block_size, d))
    _require(sel_idx, "sel_idx", torch.int32, (b, h, n // block_size, top_n))
    cfg = config_for(q, block_size, top_n, window_blocks, scale)
    if out is None:
        out = torch.empty_like(q)
    abi.bsa_fine_attention(cfg, q, k, v, gates, o_cg_block, sel_idx, out, status_word)
    return out

"""Backward pass (training) on the GPU against the fp64 oracle's backward (needs a B200).

bsa_forward_train saves the selected blocks, the branch outputs and their row
log-sum-exps; bsa_backward returns dq, dk, dv (bf16) and dgates (fp32). The
oracle differentiates the same forward with the GPU's selected blocks held
fixed. Tolerance (bf16 gradients, fp32 accumulation), per tensor and slab,
with scale = the largest |oracle gradient|: max-abs <= 2e-2 * scale and
mean-abs <= 2e-3 * scale, the forward's bf16 bounds read relative to the
gradient's size (the forward's outputs are of order one, gradients are not).

Full-size workloads are checked with a dout that is zero outside a few
sampled query blocks per slab: every gradient is then exact for the oracle
at modest cost (blocks with zero dout contribute exact zeros), while the GPU
runs its full-size launch configuration over all blocks.
"""
import numpy as np
import pytest
import torch

import oracle
import parity
from block_sparse_spherical_b200 import abi, api
from block_sparse_spherical_b200.configs import CONFIGS
from block_sparse_spherical_b200.synthetic import bf16_bits_to_f32, f32_to_bf16_bits, make_slab

pytestmark = pytest.mark.gpu

GRAD_MAX, GRAD_MEAN = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    abi.load()


def make_dout(cfg, seed, keep_blocks=None):
    """Seeded bf16 dout [B, H, N, d]; if keep_blocks is given, zero outside those query blocks."""
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((cfg.batch, cfg.heads, cfg.n_tokens, cfg.head_dim), dtype=np.float32)
    if keep_blocks is not None:
        mask = np.zeros(cfg.n_blocks, bool)
        mask[keep_blocks] = True
        x *= np.repeat(mask, cfg.block_size)[None, None, :, None]
    bits = f32_to_bf16_bits(x)
    return torch.from_numpy(bits).view(torch.bfloat16).cuda(), bf16_bits_to_f32(bits)


def check_grads(got, want, what):
    out = {}
    for name in ("dq", "dk", "dv", "dgates"):
        g = np.asarray(got[name], np.float64)
        w = want[name]
        scale = float(np.max(np.abs(w)))
        err = np.abs(g - w)
        mx, mean = float(err.max()), float(err.mean())
        assert np.all(np.isfinite(g)), f"{what} {name}: non-finite"
        if scale == 0.0:
            assert mx == 0.0, f"{what} {name}: nonzero where the oracle is zero ({mx:.3e})"
            continue
        assert mx <= GRAD_MAX * scale and mean <= GRAD_MEAN * scale, \
            f"{what} {name}: max {mx:.3e} mean {mean:.3e} scale {scale:.3e}"
        out[name] = (mx / scale, mean / scale)
    return out


def run_train(cfg, dout):
    q, k, v, g = parity.device_inputs(cfg)
    layer = api.BSATrain.from_config(cfg)
    out = layer(q, k, v, g)
    dq, dk, dv, dg = layer.backward(dout)
    torch.cuda.synchronize()
    assert layer.check_status() == 0, "forward status word set"
    assert layer.check_backward_status() == 0, "backward status word set"
    return layer, out, (dq, dk, dv, dg)


def slab_check(cfg, layer, grads, dout64, slab, what):
    b, h = divmod(slab, cfg.heads)
    s = make_slab(cfg, slab)
    idx = layer.sel_idx[b, h].cpu().numpy()
    want = oracle.backward_slab(s.q, s.k, s.v, s.gates, idx, dout64[b, h], cfg.block_size, cfg.top_n,
                                cfg.window_blocks)
    got = {"dq": parity.to_np(grads[0][b, h]), "dk": parity.to_np(grads[1][b, h]),
           "dv": parity.to_np(grads[2][b, h]), "dgates": grads[3][b, h].cpu().numpy()}
    return check_grads(got, want, f"{what} slab {slab}")


def test_training_forward_matches_forward():
    """bsa_forward_train gives bsa_forward's output and blocks bit for bit, and its saved
    branch outputs recombine into the output."""
    cfg = CONFIGS["nside32"]
    q, k, v, g = parity.device_inputs(cfg)
    ref = api.BSA.from_config(cfg)
    o1 = ref(q, k, v, g)
    layer = api.BSATrain.from_config(cfg)
    o2 = layer(q, k, v, g)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(ref.sel_idx, layer.sel_idx)
    blk = torch.arange(cfg.n_tokens, device="cuda") // cfg.block_size
    comb = (g[..., 0:1] * layer.o_cg[:, :, blk] + g[..., 1:2] * layer.o_fg.float() + g[..., 2:3] * layer.o_l.float())
    assert float((comb - o2.float()).abs().max()) <= 2e-2
    assert torch.isfinite(layer.lse_fine).all() and torch.isfinite(layer.lse_cg).all()


@pytest.mark.parametrize("name", ["nside32"])
def test_backward_parity_full(name):
    cfg = CONFIGS[name]
    dout, dout64 = make_dout(cfg, seed=101)
    layer, _, grads = run_train(cfg, dout)
    for slab in range(cfg.slabs):
        rel = slab_check(cfg, layer, grads, dout64, slab, name)
    print(f"{name}: last slab relative errors {rel}")


@pytest.mark.parametrize("name", ["nside64", "nside128", "nside256"])
def test_backward_parity_full_size_sparse_dout(name):
    cfg = CONFIGS[name]
    m = cfg.n_blocks
    keep = [0, 1, m // 3, m // 2 + 5, m - 2, m - 1]
    dout, dout64 = make_dout(cfg, seed=202, keep_blocks=keep)
    layer, _, grads = run_train(cfg, dout)
    for slab in (0, cfg.slabs - 1):
        slab_check(cfg, layer, grads, dout64, slab, name)


EDGE = {
    # name: (block, tokens, batch, heads, top_n, window)
    "single_block": (64, 64, 1, 1, 1, 1),
    "two_blocks_all_selected_w0": (64, 128, 1, 2, 2, 0),
    "ragged_m100": (64, 6400, 2, 3, 16, 1),
    "ragged_m257_w2": (64, 64 * 257, 1, 2, 16, 2),
    "m130_n64": (64, 64 * 130, 1, 2, 64, 1),
    "window_covers_all": (64, 640, 1, 2, 3, 20),
    "topn_equals_m": (64, 2048, 1, 2, 32, 1),
    "block256_nside32": (256, 12288, 1, 2, 4, 1),
    "block1024_m13_w2": (1024, 1024 * 13, 1, 1, 3, 2),
}


@pytest.mark.parametrize("name", list(EDGE))
def test_backward_edge_cases(name):
    bk, tokens, b, h, n, w = EDGE[name]
    cfg = CONFIGS["nside32"].with_(name=name, block_size=bk, tokens=tokens, batch=b, heads=h, top_n=n,
                                   window_blocks=w, seed=300 + len(name))
    dout, dout64 = make_dout(cfg, seed=7)
    layer, _, grads = run_train(cfg, dout)
    for slab in range(cfg.slabs):
        slab_check(cfg, layer, grads, dout64, slab, name)


def test_backward_key_gradients_deterministic():
    """dk and dv are owned by one key block each (no atomics): two runs agree bit for bit."""
    cfg = CONFIGS["nside32"]
    dout, _ = make_dout(cfg, seed=9)
    _, _, g1 = run_train(cfg, dout)
    _, _, g2 = run_train(cfg, dout)
    assert torch.equal(g1[1], g2[1]) and torch.equal(g1[2], g2[2]) and torch.equal(g1[3], g2[3])


def test_backward_rejects_unsupported():
    cfg = CONFIGS["tiny_nside8"]
    with pytest.raises(abi.BsaError) as e:
        abi.bsa_backward_workspace_size(abi.make_config(cfg))
    assert e.value.code == 2

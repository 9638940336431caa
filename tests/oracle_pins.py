"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each check takes the loaded oracle library (so the mutation test can run the
same checks against deliberately broken copies) and raises AssertionError on
a mismatch. The facts used:

* closed forms of the HEALPix NESTED scheme (MOSAIC note, "HEALPix spherical
  tessellation + NESTED index": N = 12 Nside^2, children of p are 4p..4p+3);
* the three reductions of BSA to dense softmax attention that follow from the
  note's BSA section: block size 1 turns the compressed branch into full
  attention, n = m turns the selection branch into full attention, a window
  that covers every block turns the local branch into full attention. Dense
  attention is taken from torch's scaled_dot_product_attention in float64 on
  the CPU, a library routine independent of the oracle;
* brute force: the top-n list against numpy's stable argsort of the logits,
  ties with constructed equal scores, uniform attention at the window edges;
* invariants of the gated combine (one-hot gates, constant values);
* the whole forward on small inputs restated as masked dense attention
  (library SDPA with block masks), a formulation the oracle does not use.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle


def sdpa64(q, k, v, scale, mask=None):
    """Dense softmax attention from torch (float64, CPU). mask: bool [Nq, Nk], True = attend."""
    tq = torch.from_numpy(np.ascontiguousarray(q, np.float64))[None, None]
    tk = torch.from_numpy(np.ascontiguousarray(k, np.float64))[None, None]
    tv = torch.from_numpy(np.ascontiguousarray(v, np.float64))[None, None]
    am = None if mask is None else torch.from_numpy(np.ascontiguousarray(mask))[None, None]
    with torch.no_grad():
        o = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, attn_mask=am, scale=scale)
    return o[0, 0].numpy()


def rand_slab(rng, n_tok, d, block, corr=True):
    m = n_tok // block
    def one():
        eps = rng.standard_normal((n_tok, d))
        if not corr:
            return eps
        u = rng.standard_normal((m, d))
        return 0.6 * eps + 0.8 * np.repeat(u, block, axis=0)
    q, k, v = one(), one(), one()
    g = 1.0 / (1.0 + np.exp(-rng.standard_normal((n_tok, 3))))
    return q, k, v, g


def close(a, b, tol, what):
    err = float(np.max(np.abs(np.asarray(a) - np.asarray(b)))) if np.size(a) else 0.0
    assert err <= tol, f"{what}: max abs err {err:.3e} > {tol:.1e}"


# ---------------------------------------------------------------- HEALPix

def nested_ancestors(nside: int, levels_up: int) -> np.ndarray:
    """Ancestor (levels_up coarser) of every NESTED pixel, by expanding children.

    Starts from the 12 base pixels and repeatedly replaces pixel p by its four
    children 4p, 4p+1, 4p+2, 4p+3, tracking which coarse pixel each fine
    pixel descends from. No integer division is used.
    """
    depth = int(round(math.log2(nside)))
    coarse_depth = depth - levels_up
    pixels = list(range(12))                      # level 0: base pixels
    owner = list(range(12))
    for level in range(depth):
        if level == coarse_depth:
            owner = list(pixels)
        nxt, nxt_owner = [], []
        for p, o in zip(pixels, owner):
            for c in range(4):
                nxt.append(4 * p + c)
                nxt_owner.append(o)
        pixels, owner = nxt, nxt_owner
    if coarse_depth == depth:
        owner = list(pixels)
    anc = np.empty(len(pixels), np.int64)
    anc[np.asarray(pixels)] = np.asarray(owner)
    return anc


def check_pool_partition_is_nested_parent(lib):
    """A block of 4^L consecutive NESTED tokens is exactly one pixel L levels up."""
    for nside, levels in ((8, 2), (8, 1), (16, 3), (4, 2)):
        anc = nested_ancestors(nside, levels)
        n_tok, block, d = 12 * nside * nside, 4 ** levels, 3
        assert len(anc) == n_tok
        x = np.repeat(anc[:, None].astype(np.float64), d, axis=1)
        xbar = oracle.pool(x, block, lib=lib)
        want = np.repeat(np.arange(n_tok // block, dtype=np.float64)[:, None], d, axis=1)
        assert np.array_equal(xbar, want), f"pool partition != parent pixels (nside {nside}, L {levels})"


def check_pool_constant_and_linear(lib):
    rng = np.random.default_rng(11)
    n_tok, d, block = 192, 5, 16
    m = n_tok // block
    c = rng.standard_normal((m, d))
    x = np.repeat(c, block, axis=0)
    close(oracle.pool(x, block, lib=lib), c, 1e-15, "pool of block-constant input")
    a, b = rng.standard_normal((n_tok, d)), rng.standard_normal((n_tok, d))
    lhs = oracle.pool(2.0 * a - 3.0 * b, block, lib=lib)
    rhs = 2.0 * oracle.pool(a, block, lib=lib) - 3.0 * oracle.pool(b, block, lib=lib)
    close(lhs, rhs, 1e-13, "pool linearity")
    # the mean of a block of 1..B in one channel is (B+1)/2
    y = np.tile(np.arange(1, block + 1, dtype=np.float64), m)[:, None]
    close(oracle.pool(y, block, lib=lib), np.full((m, 1), (block + 1) / 2.0), 1e-15, "pool of 1..B")


# ---------------------------------------------------------- dense reductions

def check_block1_compressed_is_dense(lib):
    """Block size 1: q̄ = q, k̄ = k, v̄ = v, so o_CG is full softmax attention."""
    rng = np.random.default_rng(12)
    for n_tok, d in ((40, 8), (96, 16)):
        q, k, v, _ = rand_slab(rng, n_tok, d, 1, corr=False)
        s = 1.0 / math.sqrt(d)
        qb, kb, vb = (oracle.pool(x, 1, lib=lib) for x in (q, k, v))
        r = oracle.compressed_rows(qb, kb, vb, n=3, scale=s, lib=lib)
        close(r["o_cg"], sdpa64(q, k, v, s), 1e-12, "compressed branch with block 1 vs dense")
        # non-default scale
        r = oracle.compressed_rows(qb, kb, vb, n=3, scale=0.37, lib=lib)
        close(r["o_cg"], sdpa64(q, k, v, 0.37), 1e-12, "compressed branch (scale 0.37) vs dense")


def check_full_topn_selection_is_dense(lib):
    """n = m: every block is selected, so o_FG is full softmax attention."""
    rng = np.random.default_rng(13)
    for n_tok, d, block in ((128, 8, 16), (96, 4, 8)):
        m = n_tok // block
        q, k, v, g = rand_slab(rng, n_tok, d, block)
        s = 1.0 / math.sqrt(d)
        qb, kb, vb = (oracle.pool(x, block, lib=lib) for x in (q, k, v))
        c = oracle.compressed_rows(qb, kb, vb, n=m, scale=s, lib=lib)
        assert np.all(np.isinf(c["gap"])), "gap must be +inf when n == m"
        for row in c["idx"]:
            assert sorted(row.tolist()) == list(range(m)), "n == m must select every block once"
        f = oracle.fine_rows(q, k, v, g, c["o_cg"], c["idx"], block, m, 1, scale=s,
                             want_branches=True, lib=lib)
        close(f["o_fg"], sdpa64(q, k, v, s), 1e-12, "selection branch with n = m vs dense")


def check_full_window_local_is_dense(lib):
    """A window of w >= m blocks covers the whole sequence: o_L is full attention."""
    rng = np.random.default_rng(14)
    n_tok, d, block = 96, 8, 8
    m = n_tok // block
    q, k, v, g = rand_slab(rng, n_tok, d, block)
    s = 1.0 / math.sqrt(d)
    idx = np.zeros((m, 2), np.int32)
    idx[:, 1] = 1
    o_cg = np.zeros((m, d))
    for w in (m - 1, m, 3 * m):
        f = oracle.fine_rows(q, k, v, g, o_cg, idx, block, 2, w, scale=s, want_branches=True, lib=lib)
        close(f["o_l"], sdpa64(q, k, v, s), 1e-12, f"local branch with w={w} vs dense")


# ----------------------------------------------------------------- brute force

def check_topn_against_stable_argsort(lib):
    rng = np.random.default_rng(15)
    for m, d, n in ((48, 32, 4), (30, 8, 7), (16, 4, 16), (64, 16, 1)):
        qb, kb, vb = (rng.standard_normal((m, d)) for _ in range(3))
        r = oracle.compressed_rows(qb, kb, vb, n=n, want_z=True, lib=lib)
        z = r["z"]
        order = np.argsort(-z, axis=1, kind="stable")
        assert np.array_equal(r["idx"], order[:, :n]), "top-n differs from a stable argsort"
        zs = np.take_along_axis(z, order, axis=1)
        want_gap = zs[:, n - 1] - zs[:, n] if n < m else np.full(m, np.inf)
        assert np.array_equal(r["gap"], want_gap), "gap is not z_(n) - z_(n+1)"
        # the logits themselves: rank-one check z_ij * sqrt(d) / <q̄_i, k̄_j> == 1 on a diagonal probe
        e = np.zeros((m, d)); e[:, 0] = 1.0
        r1 = oracle.compressed_rows(e, kb, vb, n=n, want_z=True, lib=lib)
        close(r1["z"], np.broadcast_to(kb[:, 0] / math.sqrt(d), (m, m)), 1e-15,
              "z with q̄ = e_0 must be k̄_j0 / sqrt(d)")


def check_topn_ties_lower_index(lib):
    d, m = 4, 8
    kb = np.zeros((m, d))
    # scores against q̄ = e_0: block scores 0,5,2,5,1,5,3,0 (three-way tie at 5)
    kb[:, 0] = [0, 5, 2, 5, 1, 5, 3, 0]
    qb = np.zeros((1, d)); qb[0, 0] = 1.0
    vb = np.zeros((m, d))
    for n, want in ((1, [1]), (2, [1, 3]), (3, [1, 3, 5]), (4, [1, 3, 5, 6]), (8, [1, 3, 5, 6, 2, 4, 0, 7])):
        qrep = np.repeat(qb, m, axis=0)
        r = oracle.compressed_rows(qrep, kb, vb, n=n, rows=(0, 1), lib=lib)
        assert r["idx"][0].tolist() == want, f"tie order n={n}: {r['idx'][0].tolist()} != {want}"
    r = oracle.compressed_rows(np.repeat(qb, m, axis=0), kb, vb, n=2, rows=(0, 1), lib=lib)
    assert r["gap"][0] == 0.0, "gap inside a tie must be 0"


def check_window_edges_uniform(lib):
    """q = 0 makes every score 0, so each branch is the plain mean of its values."""
    d, block = 2, 4
    for m, w in ((7, 1), (7, 2), (5, 0), (3, 1)):
        n_tok = m * block
        q = np.zeros((n_tok, d))
        k = np.random.default_rng(16).standard_normal((n_tok, d))
        v = np.repeat(np.arange(m, dtype=np.float64)[:, None], block, axis=0) * np.ones((1, d))
        g = np.ones((n_tok, 3))
        n = min(2, m)
        idx = np.array([[(i + 2) % m, (i + 3) % m][:n] for i in range(m)], np.int32)
        f = oracle.fine_rows(q, k, v, g, np.zeros((m, d)), idx, block, n, w, want_branches=True, lib=lib)
        for i in range(m):
            lo, hi = max(0, i - w), min(m - 1, i + w)
            want_l = np.mean(np.arange(lo, hi + 1, dtype=np.float64))
            got = f["o_l"][i * block:(i + 1) * block]
            close(got, np.full_like(got, want_l), 1e-14, f"local mean m={m} w={w} block {i}")
            want_fg = float(np.mean(idx[i].astype(np.float64)))
            got = f["o_fg"][i * block:(i + 1) * block]
            close(got, np.full_like(got, want_fg), 1e-14, f"selection mean block {i}")


# ------------------------------------------------------------------- combine

def check_gates_and_constant_values(lib):
    rng = np.random.default_rng(17)
    n_tok, d, block, n, w = 96, 8, 8, 3, 1
    m = n_tok // block
    q, k, v, g = rand_slab(rng, n_tok, d, block)
    full = oracle.forward_slab(q, k, v, g, block, n, w, lib=lib)
    parts = oracle.fine_rows(q, k, v, g, full["o_cg"], full["idx"], block, n, w, want_branches=True, lib=lib)
    close(full["out"], parts["out"], 0.0, "forward_slab vs fine_rows composition")
    cg_tok = np.repeat(full["o_cg"], block, axis=0)
    for onehot, want in (((1, 0, 0), cg_tok), ((0, 1, 0), parts["o_fg"]), ((0, 0, 1), parts["o_l"])):
        gg = np.tile(np.asarray(onehot, np.float64), (n_tok, 1))
        o = oracle.forward_slab(q, k, v, gg, block, n, w, lib=lib)["out"]
        close(o, want, 0.0, f"one-hot gate {onehot}")
    # constant values: every branch returns c, so out = (g_CG + g_FG + g_L) * c
    c = rng.standard_normal(d)
    vc = np.tile(c, (n_tok, 1))
    o = oracle.forward_slab(q, k, vc, g, block, n, w, lib=lib)["out"]
    close(o, g.sum(axis=1, keepdims=True) * c[None, :], 1e-13, "constant v")
    # the compressed output is one vector per query block
    gg = np.tile(np.asarray((1.0, 0.0, 0.0)), (n_tok, 1))
    o = oracle.forward_slab(q, k, v, gg, block, n, w, lib=lib)["out"].reshape(m, block, d)
    close(o, np.broadcast_to(o[:, :1, :], o.shape), 0.0, "o_CG constant inside a block")


def check_forced_index_permutation(lib):
    rng = np.random.default_rng(18)
    n_tok, d, block, n, w = 128, 8, 16, 4, 1
    m = n_tok // block
    q, k, v, g = rand_slab(rng, n_tok, d, block)
    base = oracle.forward_slab(q, k, v, g, block, n, w, lib=lib)
    same = oracle.forward_slab(q, k, v, g, block, n, w, forced_idx=base["idx"], lib=lib)
    close(same["out"], base["out"], 0.0, "forcing the computed indices")
    perm = base["idx"][:, ::-1].copy()
    o = oracle.forward_slab(q, k, v, g, block, n, w, forced_idx=perm, lib=lib)
    close(o["out"], base["out"], 1e-13, "selected-list permutation")
    other = np.array([[(i + 1 + t) % m for t in range(n)] for i in range(m)], np.int32)
    o2 = oracle.forward_slab(q, k, v, g, block, n, w, forced_idx=other, lib=lib)
    assert np.max(np.abs(o2["out"] - base["out"])) > 1e-3, "forced indices are ignored"


# ------------------------------------------------- whole forward, restated

def masked_dense_restatement(q, k, v, g, block, n, w, scale):
    """BSA written as three masked dense attentions (library SDPA) + combine."""
    n_tok, d = q.shape
    m = n_tok // block
    qb, kb, vb = (x.reshape(m, block, d).mean(axis=1) for x in (q, k, v))
    o_cg = sdpa64(qb, kb, vb, scale)
    z = scale * (qb @ kb.T)
    idx = np.argsort(-z, axis=1, kind="stable")[:, :n]
    blk = np.arange(n_tok) // block
    sel_mask_blocks = np.zeros((m, m), bool)
    np.put_along_axis(sel_mask_blocks, idx, True, axis=1)
    sel_mask = sel_mask_blocks[blk][:, blk]
    loc_mask = np.abs(blk[:, None] - blk[None, :]) <= w
    o_fg = sdpa64(q, k, v, scale, sel_mask)
    o_l = sdpa64(q, k, v, scale, loc_mask)
    out = g[:, :1] * o_cg[blk] + g[:, 1:2] * o_fg + g[:, 2:3] * o_l
    return out, idx


def check_forward_against_masked_dense(lib):
    rng = np.random.default_rng(19)
    for n_tok, d, block, n, w in ((768, 32, 16, 4, 1), (256, 16, 16, 5, 2), (192, 8, 4, 48, 0)):
        q, k, v, g = rand_slab(rng, n_tok, d, block)
        s = 1.0 / math.sqrt(d)
        r = oracle.forward_slab(q, k, v, g, block, n, w, scale=s, lib=lib)
        want, idx = masked_dense_restatement(q, k, v, g, block, n, w, s)
        assert np.array_equal(r["idx"], idx), "indices differ from the masked-dense restatement"
        close(r["out"], want, 1e-12, f"forward vs masked dense (N={n_tok}, B={block}, n={n}, w={w})")


# ------------------------------------------------------------------ backward

def _loss_and_forced_forward(lib, q, k, v, g, dout, block, n, w, s, idx):
    o = oracle.forward_slab(q, k, v, g, block, n, w, scale=s, forced_idx=idx, lib=lib)["out"]
    return float(np.sum(dout * o))


def check_backward_finite_differences(lib):
    """Central differences of L = sum(dout * out) through the forward oracle (selection held
    fixed by forcing its indices) against the backward oracle, for every input element."""
    rng = np.random.default_rng(20)
    for n_tok, d, block, n, w in ((24, 4, 4, 2, 1), (32, 3, 8, 4, 0)):
        q, k, v, g = rand_slab(rng, n_tok, d, block)
        dout = rng.standard_normal((n_tok, d))
        s = 1.0 / math.sqrt(d)
        idx = oracle.forward_slab(q, k, v, g, block, n, w, scale=s, lib=lib)["idx"]
        got = oracle.backward_slab(q, k, v, g, idx, dout, block, n, w, scale=s, lib=lib)
        h = 1e-5
        for name, x in (("dq", q), ("dk", k), ("dv", v), ("dgates", g)):
            num = np.zeros_like(x)
            for e in range(x.size):
                old = x.flat[e]
                x.flat[e] = old + h
                lp = _loss_and_forced_forward(lib, q, k, v, g, dout, block, n, w, s, idx)
                x.flat[e] = old - h
                lm = _loss_and_forced_forward(lib, q, k, v, g, dout, block, n, w, s, idx)
                x.flat[e] = old
                num.flat[e] = (lp - lm) / (2 * h)
            close(got[name], num, 1e-7, f"{name} vs central differences (N={n_tok}, B={block})")


def torch_masked_dense_grads(q, k, v, g, dout, block, idx, w, scale):
    """Gradients of the masked-dense restatement by torch autograd (float64, CPU): pooling by a
    mean, the compressed branch and both fine branches as library SDPA calls with block masks."""
    n_tok, d = q.shape
    m = n_tok // block
    T = lambda a: torch.tensor(np.asarray(a, np.float64), requires_grad=True)
    tq, tk, tv, tg = T(q), T(k), T(v), T(g)
    sdpa = torch.nn.functional.scaled_dot_product_attention
    qb, kb, vb = (x.reshape(m, block, d).mean(dim=1) for x in (tq, tk, tv))
    o_cg = sdpa(qb[None, None], kb[None, None], vb[None, None], scale=scale)[0, 0]
    blk = np.arange(n_tok) // block
    selb = np.zeros((m, m), bool)
    np.put_along_axis(selb, np.asarray(idx, np.int64), True, axis=1)
    sel_mask = torch.from_numpy(selb[blk][:, blk])
    loc_mask = torch.from_numpy(np.abs(blk[:, None] - blk[None, :]) <= w)
    o_fg = sdpa(tq[None, None], tk[None, None], tv[None, None], attn_mask=sel_mask[None, None], scale=scale)[0, 0]
    o_l = sdpa(tq[None, None], tk[None, None], tv[None, None], attn_mask=loc_mask[None, None], scale=scale)[0, 0]
    out = tg[:, :1] * o_cg[torch.from_numpy(blk)] + tg[:, 1:2] * o_fg + tg[:, 2:3] * o_l
    grads = torch.autograd.grad(out, (tq, tk, tv, tg), grad_outputs=torch.from_numpy(np.asarray(dout, np.float64)))
    return {name: x.numpy() for name, x in zip(("dq", "dk", "dv", "dgates"), grads)}


def check_backward_against_autograd(lib):
    """The backward oracle against torch autograd of the masked-dense restatement, including a
    dout that is zero outside a few query blocks (the oracle skips those blocks)."""
    rng = np.random.default_rng(21)
    for n_tok, d, block, n, w, sparse in ((256, 16, 16, 5, 1, False), (192, 8, 4, 48, 0, False),
                                          (384, 8, 16, 3, 2, True)):
        q, k, v, g = rand_slab(rng, n_tok, d, block)
        s = 1.0 / math.sqrt(d)
        dout = rng.standard_normal((n_tok, d))
        if sparse:
            keep = np.zeros(n_tok // block, bool)
            keep[[1, 7, n_tok // block - 1]] = True
            dout *= np.repeat(keep, block)[:, None]
        idx = oracle.forward_slab(q, k, v, g, block, n, w, scale=s, lib=lib)["idx"]
        got = oracle.backward_slab(q, k, v, g, idx, dout, block, n, w, scale=s, lib=lib)
        want = torch_masked_dense_grads(q, k, v, g, dout, block, idx, w, s)
        for name in ("dq", "dk", "dv", "dgates"):
            close(got[name], want[name], 1e-11, f"{name} vs autograd (N={n_tok}, n={n}, w={w}, sparse={sparse})")


def check_backward_linear_in_dout_and_gates(lib):
    """Gradients are linear in dout; dgates equals dout against each branch's forward output."""
    rng = np.random.default_rng(22)
    n_tok, d, block, n, w = 128, 8, 16, 3, 1
    q, k, v, g = rand_slab(rng, n_tok, d, block)
    s = 1.0 / math.sqrt(d)
    fwd = oracle.forward_slab(q, k, v, g, block, n, w, scale=s, lib=lib)
    a, b = rng.standard_normal((n_tok, d)), rng.standard_normal((n_tok, d))
    ga = oracle.backward_slab(q, k, v, g, fwd["idx"], a, block, n, w, scale=s, lib=lib)
    gb = oracle.backward_slab(q, k, v, g, fwd["idx"], b, block, n, w, scale=s, lib=lib)
    gab = oracle.backward_slab(q, k, v, g, fwd["idx"], 2 * a - 3 * b, block, n, w, scale=s, lib=lib)
    for name in ("dq", "dk", "dv", "dgates"):
        close(gab[name], 2 * ga[name] - 3 * gb[name], 1e-12, f"{name} linear in dout")
    parts = oracle.fine_rows(q, k, v, g, fwd["o_cg"], fwd["idx"], block, n, w, scale=s, want_branches=True, lib=lib)
    cg_tok = np.repeat(fwd["o_cg"], block, axis=0)
    want = np.stack([np.sum(a * cg_tok, 1), np.sum(a * parts["o_fg"], 1), np.sum(a * parts["o_l"], 1)], 1)
    close(ga["dgates"], want, 1e-13, "dgates = dout against the branch outputs")
    zero = oracle.backward_slab(q, k, v, g, fwd["idx"], np.zeros((n_tok, d)), block, n, w, scale=s, lib=lib)
    for name in ("dq", "dk", "dv", "dgates"):
        assert not np.any(zero[name]), f"{name} must vanish for dout = 0"


# ------------------------------------------- lat-lon -> HEALPix interpolation

def ring_scheme_centres(nside):
    """Pixel centres listed ring by ring (the published HEALPix ring formulas), no faces or bits."""
    pts = []
    for i in range(1, 4 * nside):
        if i < nside:
            nr, z, s = i, 1 - i * i / (3 * nside * nside), 1
        elif i > 3 * nside:
            nr = 4 * nside - i
            z, s = -1 + nr * nr / (3 * nside * nside), 1
        else:
            nr, z, s = nside, 4 / 3 - 2 * i / (3 * nside), (i - nside + 1) % 2
        for j in range(1, 4 * nr + 1):
            pts.append((z, ((j - s / 2) * math.pi / (2 * nr)) % (2 * math.pi)))
    return np.array(pts)


def unit(zphi):
    z, ph = zphi[:, 0], zphi[:, 1]
    assert np.all(np.isfinite(zphi)) and np.all(np.abs(z) <= 1), "a point off the sphere (|z| > 1 or not finite)"
    st = np.sqrt(1 - z * z)
    return np.stack([st * np.cos(ph), st * np.sin(ph), z], 1)


def check_healpix_centres(lib):
    """NESTED centres: the 12 base pixels, the same point set as the ring-by-ring listing, equal
    area (mean z^2 of a uniform sphere sample tends to 1/3), and the child rule 4p..4p+3 (the
    four children of p surround p's centre)."""
    c1 = oracle.healpix_centers(1, lib=lib)
    want_z = [2 / 3] * 4 + [0] * 4 + [-2 / 3] * 4
    want_phi = [math.pi / 4 * (2 * f + 1) for f in range(4)] + [math.pi / 2 * f for f in range(4)] + \
               [math.pi / 4 * (2 * f + 1) for f in range(4)]
    close(c1[:, 0], want_z, 1e-15, "base pixel z")
    close(c1[:, 1], want_phi, 1e-15, "base pixel phi")
    for nside in (2, 4, 8, 16):
        c = oracle.healpix_centers(nside, lib=lib)
        assert len(c) == 12 * nside * nside
        key = lambda a: sorted((round(z, 12), round(p, 12)) for z, p in a)
        assert key(c) == key(ring_scheme_centres(nside)), f"centres differ from the ring listing (nside {nside})"
        assert abs(float(np.mean(c[:, 0] ** 2)) - 1 / 3) < 0.2 / nside ** 2 + 1e-3
        fine = unit(oracle.healpix_centers(2 * nside, lib=lib)).reshape(-1, 4, 3)
        parent = unit(c)
        mean_child = fine.mean(axis=1)
        mean_child /= np.linalg.norm(mean_child, axis=1, keepdims=True)
        ang = np.degrees(np.arccos(np.clip(np.sum(mean_child * parent, 1), -1, 1)))
        assert ang.max() < 0.5 * 58.63 / nside, f"children 4p..4p+3 not around p (nside {nside}: {ang.max():.2f} deg)"


def check_latlon_plan(lib):
    """Every neighbourhood holds 16 distinct grid points including the target's nearest grid point
    (brute force over the whole grid), and the relative positions are the unit-vector differences
    over the grid step."""
    for nside, nlat, nlon in ((4, 25, 48), (8, 19, 36), (2, 7, 12)):
        nbr, rel = oracle.latlon_plan(nside, nlat, nlon, lib=lib)
        tgt = unit(oracle.healpix_centers(nside, lib=lib))
        dlat = 180 / (nlat - 1)
        lat = np.radians(90 - dlat * np.arange(nlat))
        lon = np.radians(360 / nlon * np.arange(nlon))
        src = np.stack([np.cos(lat)[:, None] * np.cos(lon)[None, :], np.cos(lat)[:, None] * np.sin(lon)[None, :],
                        np.broadcast_to(np.sin(lat)[:, None], (nlat, nlon))], -1).reshape(-1, 3)
        nearest = np.argmax(tgt @ src.T, axis=1)
        for i in range(len(tgt)):
            assert len(set(nbr[i].tolist())) == 16, f"pixel {i}: repeated neighbours"
            assert nearest[i] in set(nbr[i].tolist()) or np.isclose(
                (tgt[i] @ src[nearest[i]]), max(tgt[i] @ src[j] for j in nbr[i]), atol=1e-12), \
                f"pixel {i}: nearest grid point not in its neighbourhood"
        close(rel, (src[nbr] - tgt[:, None, :]) / np.radians(dlat), 1e-12, "relative positions")


def check_interp(lib):
    """The interpolation against (a) the logits formed the other way round, q_ij . k_j =
    p_ij . (W_q^T k_j), with a library softmax; (b) W_q = 0: the plain mean of the neighbours'
    values; (c) one neighbour set repeated: the value itself."""
    rng = np.random.default_rng(23)
    n_src, d, K, n_tgt = 40, 16, 16, 30
    nbr = np.stack([rng.choice(n_src, K, replace=False) for _ in range(n_tgt)]).astype(np.int32)
    rel = rng.standard_normal((n_tgt, K, 3))
    wq = rng.standard_normal((d, 3))
    ks, vs = rng.standard_normal((n_src, d)), rng.standard_normal((n_src, d))
    s = 1 / math.sqrt(d)
    got = oracle.interp(nbr, rel, wq, ks, vs, lib=lib)
    kappa = ks @ wq                                   # [n_src, 3]: keys seen from position space
    logits = s * np.einsum("ike,ike->ik", rel, kappa[nbr])
    p = torch.softmax(torch.from_numpy(logits), dim=1).numpy()
    close(got, np.einsum("ik,ikc->ic", p, vs[nbr]), 1e-13, "interp vs position-space logits")
    close(oracle.interp(nbr, rel, np.zeros((d, 3)), ks, vs, lib=lib), vs[nbr].mean(axis=1), 1e-14, "W_q = 0 mean")
    one = np.repeat(nbr[:, :1], K, axis=1)
    close(oracle.interp(one, rel, wq, ks, vs, lib=lib), vs[nbr[:, 0]], 1e-14, "single source")


ALL_CHECKS = [
    check_pool_partition_is_nested_parent,
    check_pool_constant_and_linear,
    check_block1_compressed_is_dense,
    check_full_topn_selection_is_dense,
    check_full_window_local_is_dense,
    check_topn_against_stable_argsort,
    check_topn_ties_lower_index,
    check_window_edges_uniform,
    check_gates_and_constant_values,
    check_forced_index_permutation,
    check_forward_against_masked_dense,
    check_backward_finite_differences,
    check_backward_against_autograd,
    check_backward_linear_in_dout_and_gates,
    check_healpix_centres,
    check_latlon_plan,
    check_interp,
]

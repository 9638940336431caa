// C ABI of the BSA forward pass (declared in include/bsa.h): argument
// validation, workspace layout and kernel dispatch. No allocation, no
// synchronisation (except bsa_check_status), no global state.
#include <math.h>
#include <stdint.h>

#include "bsa_internal.cuh"
#include "bsa_testing.h"

namespace {

using bsa::Problem;

constexpr size_t kAlign = 256;
size_t round_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// bf16: blocks of 64, 256 or 1024 tokens (a parent pixel 3, 4 or 5 levels up), head_dim 64, on
// the tensor cores; fp32: (16, 32) and (64, 64) on the CUDA cores.
bool shape_supported(int32_t dtype, int32_t bk, int32_t d) {
    return (dtype == BSA_BF16 && (bk == 64 || bk == 256 || bk == 1024) && d == 64) ||
           (dtype == BSA_F32 && bk == 64 && d == 64) || (dtype == BSA_F32 && bk == 16 && d == 32);
}

bsa_status make_problem(const bsa_config *cfg, Problem *p) {
    if (!cfg) return BSA_ERR_INVALID_ARG;
    if (cfg->batch < 1 || cfg->heads < 1 || cfg->n_tokens < 1 || cfg->head_dim < 1 || cfg->block_size < 1)
        return BSA_ERR_INVALID_ARG;
    if (cfg->n_tokens % cfg->block_size != 0) return BSA_ERR_INVALID_ARG;
    const int64_t m = cfg->n_tokens / cfg->block_size;
    if (cfg->top_n < 1 || cfg->top_n > m || cfg->window_blocks < 0) return BSA_ERR_INVALID_ARG;
    if (cfg->dtype != BSA_F32 && cfg->dtype != BSA_BF16) return BSA_ERR_INVALID_ARG;
    if (!(cfg->scale >= 0.0f) || isinf(cfg->scale)) return BSA_ERR_INVALID_ARG;
    if (!shape_supported(cfg->dtype, cfg->block_size, cfg->head_dim)) return BSA_ERR_UNSUPPORTED;
    if (cfg->top_n > bsa::kMaxTopN) return BSA_ERR_UNSUPPORTED;
    const int64_t slabs = (int64_t)cfg->batch * cfg->heads;
    if (slabs > 65535) return BSA_ERR_UNSUPPORTED;            // grid.y of the per-slab kernels
    // the tensor-core kernel addresses token rows with 32-bit TMA coordinates
    if (cfg->dtype == BSA_BF16 && slabs * cfg->n_tokens > 0x7fffffffLL) return BSA_ERR_UNSUPPORTED;
    p->batch = cfg->batch;
    p->heads = cfg->heads;
    p->n_tokens = cfg->n_tokens;
    p->head_dim = cfg->head_dim;
    p->block_size = cfg->block_size;
    p->top_n = cfg->top_n;
    p->window = cfg->window_blocks;
    p->m = m;
    p->slabs = slabs;
    p->dtype = (bsa_dtype)cfg->dtype;
    p->scale = cfg->scale > 0.0f ? cfg->scale : 1.0f / sqrtf((float)cfg->head_dim);
    return BSA_OK;
}

struct WorkspaceLayout {
    size_t status, qbar, kbar, vbar, o_cg, idx;
    size_t base;      // end of the above (what the allocation-free entry point needs)
    size_t split;     // tf32 split images of the tensor-core compressed kernel (0 bytes if unused)
    size_t total;
};

WorkspaceLayout layout_of(const Problem &p) {
    const size_t pooled = (size_t)p.slabs * p.m * p.head_dim * sizeof(float);
    const size_t idx = (size_t)p.slabs * p.m * p.top_n * sizeof(int32_t);
    WorkspaceLayout w;
    w.status = 0;
    w.qbar = kAlign;
    w.kbar = w.qbar + round_up(pooled);
    w.vbar = w.kbar + round_up(pooled);
    w.o_cg = w.vbar + round_up(pooled);
    w.idx = w.o_cg + round_up(pooled);
    w.base = w.idx + round_up(idx);
    w.split = w.base;
    w.total = w.split + round_up(bsa::compress_tc_workspace_bytes(p));
    return w;
}

bsa_status from_cuda(cudaError_t e) {
    if (e == cudaSuccess) return BSA_OK;
    if (e == cudaErrorNotSupported) return BSA_ERR_UNSUPPORTED;
    return BSA_ERR_CUDA;
}

// Compressed branch + top-n: the tensor-core kernel where it takes the shape
// (with its split images in `images` when given), else the CUDA-core kernel.
cudaError_t launch_compress(const Problem &p, const float *qbar, const float *kbar, const float *vbar,
                            float *o_cg, int32_t *idx, uint32_t *status, void *images, cudaStream_t stream) {
    const cudaError_t e = bsa::launch_compress_tc(p, qbar, kbar, vbar, o_cg, idx, status, images, stream);
    if (e != cudaErrorNotSupported) return e;
    return bsa::launch_compress_select(p, qbar, kbar, vbar, o_cg, idx, stream);
}

// Selection + local branches and the combine: bf16 problems run on the tensor cores only (a
// failure there is returned, never retried elsewhere); fp32 problems on the CUDA cores.
cudaError_t launch_fine(const Problem &p, const void *q, const void *k, const void *v,
                        const float *gates, const float *o_cg, const int32_t *idx, void *out,
                        uint32_t *status, cudaStream_t stream) {
    if (p.dtype == BSA_BF16) return bsa::launch_attend_tc(p, q, k, v, gates, o_cg, idx, out, status, stream);
    return bsa::launch_attend_simt(p, q, k, v, gates, o_cg, idx, out, status, stream);
}

}  // namespace

extern "C" {

bsa_status bsa_pool(const bsa_config *cfg, const void *q, const void *k, const void *v,
                    float *qbar, float *kbar, float *vbar, cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!q || !k || !v || !qbar || !kbar || !vbar) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(qbar) || !aligned16(kbar) ||
        !aligned16(vbar))
        return BSA_ERR_ALIGNMENT;
    return from_cuda(bsa::launch_pool(p, q, k, v, qbar, kbar, vbar, stream));
}

bsa_status bsa_compress_select(const bsa_config *cfg, const float *qbar, const float *kbar,
                               const float *vbar, float *o_cg_block, int32_t *sel_idx,
                               cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!qbar || !kbar || !vbar || !o_cg_block || !sel_idx) return BSA_ERR_INVALID_ARG;
    if (!aligned16(qbar) || !aligned16(kbar) || !aligned16(vbar) || !aligned16(o_cg_block) ||
        !aligned16(sel_idx))
        return BSA_ERR_ALIGNMENT;
    return from_cuda(launch_compress(p, qbar, kbar, vbar, o_cg_block, sel_idx, nullptr, nullptr, stream));
}

bsa_status bsa_compress_select_ws(const bsa_config *cfg, const float *qbar, const float *kbar,
                                  const float *vbar, float *o_cg_block, int32_t *sel_idx, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!qbar || !kbar || !vbar || !o_cg_block || !sel_idx) return BSA_ERR_INVALID_ARG;
    if (!workspace) return BSA_ERR_WORKSPACE;
    const WorkspaceLayout L = layout_of(p);
    if (workspace_bytes < L.total) return BSA_ERR_WORKSPACE;
    if (!aligned16(qbar) || !aligned16(kbar) || !aligned16(vbar) || !aligned16(o_cg_block) ||
        !aligned16(sel_idx) || ((uintptr_t)workspace & (kAlign - 1)))
        return BSA_ERR_ALIGNMENT;
    void *images = L.total > L.split ? static_cast<char *>(workspace) + L.split : nullptr;
    return from_cuda(launch_compress(p, qbar, kbar, vbar, o_cg_block, sel_idx, nullptr, images, stream));
}

bsa_status bsa_fine_attention(const bsa_config *cfg, const void *q, const void *k, const void *v,
                              const float *gates, const float *o_cg_block, const int32_t *sel_idx,
                              void *out, uint32_t *status_word, cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!q || !k || !v || !gates || !o_cg_block || !sel_idx || !out) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gates) || !aligned16(o_cg_block) ||
        !aligned16(sel_idx) || !aligned16(out) || ((uintptr_t)status_word & 3u))
        return BSA_ERR_ALIGNMENT;
    return from_cuda(launch_fine(p, q, k, v, gates, o_cg_block, sel_idx, out, status_word, stream));
}

bsa_status bsa_workspace_size(const bsa_config *cfg, size_t *bytes) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!bytes) return BSA_ERR_INVALID_ARG;
    *bytes = layout_of(p).total;
    return BSA_OK;
}

bsa_status bsa_forward(const bsa_config *cfg, const void *q, const void *k, const void *v,
                       const float *gates, void *out, int32_t *sel_idx_out, void *workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!q || !k || !v || !gates || !out) return BSA_ERR_INVALID_ARG;
    if (!workspace) return BSA_ERR_WORKSPACE;
    const WorkspaceLayout L = layout_of(p);
    if (workspace_bytes < L.total) return BSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gates) || !aligned16(out) ||
        !aligned16(sel_idx_out) || ((uintptr_t)workspace & (kAlign - 1)))
        return BSA_ERR_ALIGNMENT;
    char *ws = static_cast<char *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws + L.status);
    float *qbar = reinterpret_cast<float *>(ws + L.qbar);
    float *kbar = reinterpret_cast<float *>(ws + L.kbar);
    float *vbar = reinterpret_cast<float *>(ws + L.vbar);
    float *ocg = reinterpret_cast<float *>(ws + L.o_cg);
    int32_t *idx = sel_idx_out ? sel_idx_out : reinterpret_cast<int32_t *>(ws + L.idx);
    cudaError_t e = bsa::launch_pool(p, q, k, v, qbar, kbar, vbar, stream);
    void *images = L.total > L.split ? ws + L.split : nullptr;
    if (e == cudaSuccess) e = launch_compress(p, qbar, kbar, vbar, ocg, idx, status, images, stream);
    if (e == cudaSuccess) e = launch_fine(p, q, k, v, gates, ocg, idx, out, status, stream);
    return from_cuda(e);
}

// ---- training: forward with saved tensors, and the backward ---------------

namespace {

bool train_supported(const Problem &p) { return p.dtype == BSA_BF16 && p.head_dim == 64; }

struct BwdLayout {
    size_t status, qbar, kbar, vbar, dfine, docg16, q16, k16, v16, dcg, lse_pad, dqbar, dkbar, dvbar;
    size_t count, offs, cursor, list_tmp, list, total;
    int64_t m_pad;
};

BwdLayout bwd_layout_of(const Problem &p) {
    BwdLayout L;
    L.m_pad = (p.m + 63) / 64 * 64;
    const size_t pooled = (size_t)p.slabs * p.m * p.head_dim * sizeof(float);
    const size_t pad16 = (size_t)p.slabs * L.m_pad * p.head_dim * 2, pad32 = 2 * pad16;
    const size_t pad1 = (size_t)p.slabs * L.m_pad * sizeof(float);
    const size_t rows = (size_t)p.slabs * p.n_tokens;
    const size_t ints_m = (size_t)p.slabs * p.m * sizeof(int), ints_list = ints_m * p.top_n;
    size_t o = 0;
    auto take = [&](size_t bytes) { const size_t at = o; o += round_up(bytes); return at; };
    L.status = take(kAlign);
    L.qbar = take(pooled);
    L.kbar = take(pooled);
    L.vbar = take(pooled);
    L.dfine = take(rows * 2 * sizeof(float));
    L.docg16 = take(pad16);
    L.q16 = take(pad16);
    L.k16 = take(pad16);
    L.v16 = take(pad16);
    L.dcg = take(pad1);
    L.lse_pad = take(pad1);
    L.dqbar = take(pad32);
    L.dkbar = take(pad32);
    L.dvbar = take(pad32);
    L.count = take(ints_m);
    L.offs = take((size_t)p.slabs * (p.m + 1) * sizeof(int));
    L.cursor = take(ints_m);
    L.list_tmp = take(ints_list);
    L.list = take(ints_list);
    L.total = o;
    return L;
}

}  // namespace

bsa_status bsa_forward_train(const bsa_config *cfg, const void *q, const void *k, const void *v,
                             const float *gates, void *out, int32_t *sel_idx, float *o_cg_block, float *lse_cg,
                             void *o_fg, void *o_l, float *lse_fine, void *workspace, size_t workspace_bytes,
                             cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!train_supported(p)) return BSA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gates || !out || !sel_idx || !o_cg_block || !lse_cg || !o_fg || !o_l || !lse_fine)
        return BSA_ERR_INVALID_ARG;
    if (!workspace) return BSA_ERR_WORKSPACE;
    const WorkspaceLayout L = layout_of(p);
    if (workspace_bytes < L.total) return BSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gates) || !aligned16(out) ||
        !aligned16(sel_idx) || !aligned16(o_cg_block) || !aligned16(lse_cg) || !aligned16(o_fg) ||
        !aligned16(o_l) || !aligned16(lse_fine) || ((uintptr_t)workspace & (kAlign - 1)))
        return BSA_ERR_ALIGNMENT;
    char *ws = static_cast<char *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws + L.status);
    float *qbar = reinterpret_cast<float *>(ws + L.qbar);
    float *kbar = reinterpret_cast<float *>(ws + L.kbar);
    float *vbar = reinterpret_cast<float *>(ws + L.vbar);
    void *images = L.total > L.split ? ws + L.split : nullptr;
    cudaError_t e = bsa::launch_pool(p, q, k, v, qbar, kbar, vbar, stream);
    if (e == cudaSuccess) {
        e = bsa::launch_compress_tc(p, qbar, kbar, vbar, o_cg_block, sel_idx, status, images, stream, lse_cg);
        if (e == cudaErrorNotSupported)
            e = bsa::launch_compress_select(p, qbar, kbar, vbar, o_cg_block, sel_idx, stream, lse_cg);
    }
    if (e == cudaSuccess)
        e = bsa::launch_attend_tc(p, q, k, v, gates, o_cg_block, sel_idx, out, status, stream, o_fg, o_l, lse_fine);
    return from_cuda(e);
}

bsa_status bsa_backward_workspace_size(const bsa_config *cfg, size_t *bytes) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!train_supported(p)) return BSA_ERR_UNSUPPORTED;
    if (!bytes) return BSA_ERR_INVALID_ARG;
    *bytes = bwd_layout_of(p).total;
    return BSA_OK;
}

bsa_status bsa_backward(const bsa_config *cfg, const void *q, const void *k, const void *v, const float *gates,
                        const void *dout, const int32_t *sel_idx, const float *o_cg_block, const float *lse_cg,
                        const void *o_fg, const void *o_l, const float *lse_fine, void *dq, void *dk, void *dv,
                        float *dgates, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!train_supported(p)) return BSA_ERR_UNSUPPORTED;
    const void *in[] = {q, k, v, gates, dout, sel_idx, o_cg_block, lse_cg, o_fg, o_l, lse_fine, dq, dk, dv, dgates};
    for (const void *x : in)
        if (!x) return BSA_ERR_INVALID_ARG;
    if (!workspace) return BSA_ERR_WORKSPACE;
    const BwdLayout L = bwd_layout_of(p);
    if (workspace_bytes < L.total) return BSA_ERR_WORKSPACE;
    for (const void *x : in)
        if (!aligned16(x)) return BSA_ERR_ALIGNMENT;
    if ((uintptr_t)workspace & (kAlign - 1)) return BSA_ERR_ALIGNMENT;
    char *ws = static_cast<char *>(workspace);
    bsa::BwdBuffers b;
    b.q = q; b.k = k; b.v = v; b.dout = dout; b.gates = gates; b.sel_idx = sel_idx;
    b.o_cg = o_cg_block; b.lse_cg = lse_cg; b.o_fg = o_fg; b.o_l = o_l; b.lse_fine = lse_fine;
    b.dq = dq; b.dk = dk; b.dv = dv; b.dgates = dgates;
    b.m_pad = L.m_pad;
    b.status = reinterpret_cast<uint32_t *>(ws + L.status);
    b.qbar = reinterpret_cast<float *>(ws + L.qbar);
    b.kbar = reinterpret_cast<float *>(ws + L.kbar);
    b.vbar = reinterpret_cast<float *>(ws + L.vbar);
    b.dfine = reinterpret_cast<float *>(ws + L.dfine);
    b.docg16 = ws + L.docg16;
    b.q16 = ws + L.q16;
    b.k16 = ws + L.k16;
    b.v16 = ws + L.v16;
    b.dcg = reinterpret_cast<float *>(ws + L.dcg);
    b.lse_cg_pad = reinterpret_cast<float *>(ws + L.lse_pad);
    b.dqbar = reinterpret_cast<float *>(ws + L.dqbar);
    b.dkbar = reinterpret_cast<float *>(ws + L.dkbar);
    b.dvbar = reinterpret_cast<float *>(ws + L.dvbar);
    b.count = reinterpret_cast<int *>(ws + L.count);
    b.offs = reinterpret_cast<int *>(ws + L.offs);
    b.cursor = reinterpret_cast<int *>(ws + L.cursor);
    b.list_tmp = reinterpret_cast<int *>(ws + L.list_tmp);
    b.list = reinterpret_cast<int *>(ws + L.list);
    // the pooled dq̄ is reduced into from every key tile of the compressed pass: it starts at zero
    // (a memset, not an allocation)
    cudaError_t e = cudaMemsetAsync(ws + L.dqbar, 0, (size_t)p.slabs * L.m_pad * p.head_dim * 4, stream);
    if (e == cudaSuccess) e = bsa::launch_pool(p, q, k, v, b.qbar, b.kbar, b.vbar, stream);
    if (e == cudaSuccess) e = bsa::launch_bwd_prep(p, b, stream);
    if (e == cudaSuccess) e = bsa::launch_attend_bwd_compressed(p, b, stream);
    if (e == cudaSuccess)
        e = bsa::launch_inverse_index(p, sel_idx, b.count, b.offs, b.cursor, b.list_tmp, b.list, b.status, stream);
    if (e == cudaSuccess) e = bsa::launch_attend_bwd_fine(p, b, stream);   // dk, dv, then dq
    return from_cuda(e);
}

bsa_status bsa_permute_tokens(int64_t slabs, int64_t n_tokens, int64_t row_bytes, const int32_t *perm,
                              const void *src, void *dst, uint32_t *status_word, cudaStream_t stream) {
    if (slabs < 1 || n_tokens < 1 || n_tokens > 0x7fffffffLL || row_bytes < 4 || row_bytes % 4 != 0 ||
        row_bytes / 4 > 0x7fffffffLL)
        return BSA_ERR_INVALID_ARG;
    if (!perm || !src || !dst) return BSA_ERR_INVALID_ARG;
    if (src == dst) return BSA_ERR_INVALID_ARG;        // rows move between two distinct buffers
    const uintptr_t need = row_bytes % 16 == 0 ? 15u : 3u;
    if (((uintptr_t)src & need) || ((uintptr_t)dst & need) || ((uintptr_t)perm & 3u) || ((uintptr_t)status_word & 3u))
        return BSA_ERR_ALIGNMENT;
    return from_cuda(bsa::launch_permute_rows(src, dst, perm, slabs, n_tokens, row_bytes, status_word, stream));
}

bsa_status bsa_latlon_healpix_plan(int64_t nside, int64_t nlat, int64_t nlon, int32_t *nbr, float *rel,
                                   cudaStream_t stream) {
    if (nside < 1 || nside > (1 << 13) || (nside & (nside - 1)) || nlat < 4 || nlon < 4 ||
        (int64_t)nlat * nlon > 0x7fffffffLL)
        return BSA_ERR_INVALID_ARG;
    if (!nbr || !rel) return BSA_ERR_INVALID_ARG;
    if (((uintptr_t)nbr & 15u) || ((uintptr_t)rel & 15u)) return BSA_ERR_ALIGNMENT;
    return from_cuda(bsa::launch_healpix_plan(nside, nlat, nlon, nbr, rel, stream));
}

bsa_status bsa_latlon_workspace_size(int64_t batch, int64_t n_src, size_t *bytes) {
    if (batch < 1 || n_src < 1 || !bytes) return BSA_ERR_INVALID_ARG;
    *bytes = round_up((size_t)batch * n_src * 3 * sizeof(float));
    return BSA_OK;
}

bsa_status bsa_latlon_to_healpix(int64_t batch, int64_t n_tgt, int64_t n_src, int64_t head_dim, int32_t dtype,
                                 float scale, const int32_t *nbr, const float *rel, const float *wq,
                                 const void *k_src, const void *v_src, void *out, void *workspace,
                                 size_t workspace_bytes, uint32_t *status_word, cudaStream_t stream) {
    if (batch < 1 || batch > 65535 || n_tgt < 1 || n_src < 1 || n_src > 0x7fffffffLL) return BSA_ERR_INVALID_ARG;
    if (!workspace || workspace_bytes < (size_t)batch * n_src * 3 * sizeof(float)) return BSA_ERR_WORKSPACE;
    if (dtype != BSA_F32 && dtype != BSA_BF16) return BSA_ERR_INVALID_ARG;
    if (!(scale >= 0.0f) || isinf(scale)) return BSA_ERR_INVALID_ARG;
    if (head_dim != 32 && head_dim != 64 && head_dim != 128) return BSA_ERR_UNSUPPORTED;
    if (!nbr || !rel || !wq || !k_src || !v_src || !out) return BSA_ERR_INVALID_ARG;
    if (!aligned16(nbr) || !aligned16(rel) || !aligned16(wq) || !aligned16(k_src) || !aligned16(v_src) ||
        !aligned16(out) || !aligned16(workspace) || ((uintptr_t)status_word & 3u))
        return BSA_ERR_ALIGNMENT;
    const float s = scale > 0.0f ? scale : 1.0f / sqrtf((float)head_dim);
    return from_cuda(bsa::launch_interp(batch, n_tgt, n_src, head_dim, (bsa_dtype)dtype, nbr, rel, wq, k_src, v_src,
                                        out, s, static_cast<float *>(workspace), status_word, stream));
}

bsa_status bsa_forward_mirrored(const bsa_config *cfg, const void *q, const void *k, const void *v,
                                const float *gates, void *out, void *const *mirrors, int32_t n_mirrors,
                                int32_t *sel_idx_out, void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (p.dtype != BSA_BF16) return BSA_ERR_UNSUPPORTED;
    if (!q || !k || !v || !gates || !out || n_mirrors < 0 || n_mirrors > 7 || (n_mirrors > 0 && !mirrors))
        return BSA_ERR_INVALID_ARG;
    for (int i = 0; i < n_mirrors; ++i) {
        if (!mirrors[i] || mirrors[i] == out) return BSA_ERR_INVALID_ARG;
        if (!aligned16(mirrors[i])) return BSA_ERR_ALIGNMENT;
    }
    if (!workspace) return BSA_ERR_WORKSPACE;
    const WorkspaceLayout L = layout_of(p);
    if (workspace_bytes < L.total) return BSA_ERR_WORKSPACE;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gates) || !aligned16(out) ||
        !aligned16(sel_idx_out) || ((uintptr_t)workspace & (kAlign - 1)))
        return BSA_ERR_ALIGNMENT;
    char *ws = static_cast<char *>(workspace);
    uint32_t *status = reinterpret_cast<uint32_t *>(ws + L.status);
    float *qbar = reinterpret_cast<float *>(ws + L.qbar);
    float *kbar = reinterpret_cast<float *>(ws + L.kbar);
    float *vbar = reinterpret_cast<float *>(ws + L.vbar);
    float *ocg = reinterpret_cast<float *>(ws + L.o_cg);
    int32_t *idx = sel_idx_out ? sel_idx_out : reinterpret_cast<int32_t *>(ws + L.idx);
    void *images = L.total > L.split ? ws + L.split : nullptr;
    cudaError_t e = bsa::launch_pool(p, q, k, v, qbar, kbar, vbar, stream);
    if (e == cudaSuccess) e = launch_compress(p, qbar, kbar, vbar, ocg, idx, status, images, stream);
    if (e == cudaSuccess)
        e = bsa::launch_attend_tc(p, q, k, v, gates, ocg, idx, out, status, stream, nullptr, nullptr, nullptr, mirrors,
                                  n_mirrors);
    return from_cuda(e);
}

bsa_status bsa_check_status(const void *status_word, cudaStream_t stream) {
    if (!status_word || ((uintptr_t)status_word & 3u)) return BSA_ERR_INVALID_ARG;
    uint32_t word = 0;
    if (cudaStreamSynchronize(stream) != cudaSuccess) return BSA_ERR_CUDA;
    if (cudaMemcpy(&word, status_word, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess)
        return BSA_ERR_CUDA;
    if (word != 0) {
        if (cudaMemsetAsync(const_cast<void *>(status_word), 0, sizeof(word), stream) != cudaSuccess ||
            cudaStreamSynchronize(stream) != cudaSuccess)
            return BSA_ERR_CUDA;
    }
    if (word & bsa::kStatusTimeout) return BSA_ERR_TIMEOUT;
    if (word & bsa::kStatusBadIndex) return BSA_ERR_INDEX;
    return BSA_OK;
}

const char *bsa_status_string(bsa_status s) {
    switch (s) {
        case BSA_OK: return "BSA_OK";
        case BSA_ERR_INVALID_ARG: return "BSA_ERR_INVALID_ARG: invalid argument";
        case BSA_ERR_UNSUPPORTED: return "BSA_ERR_UNSUPPORTED: shape or dtype not compiled";
        case BSA_ERR_ALIGNMENT: return "BSA_ERR_ALIGNMENT: pointer not 16-byte aligned";
        case BSA_ERR_CUDA: return "BSA_ERR_CUDA: CUDA runtime or launch failure";
        case BSA_ERR_TIMEOUT: return "BSA_ERR_TIMEOUT: a kernel's bounded wait expired";
        case BSA_ERR_WORKSPACE: return "BSA_ERR_WORKSPACE: workspace missing or too small";
        case BSA_ERR_INDEX: return "BSA_ERR_INDEX: block index outside [0, m)";
    }
    return "BSA_ERR_UNKNOWN";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward pass.
//
// Some callers cannot call cudaMalloc at the point where they run BSA: code
// that executes inside a host callback or another library's allocator hook,
// plugins whose host framework owns every device allocation, or services
// that must not touch the allocator on the request path. For them,
// bsa_forward_noalloc computes what bsa_forward computes but keeps the
// intermediates (pooled q̄/k̄/v̄, block-level compressed output, block
// indices) in a fixed array of device memory that this library owns; its
// compressed branch splits operands in every CTA (no space for split images).
//
// The array lives in device global memory for as long as the library is
// loaded, on every GPU that loads it, and is shared by every call on that
// GPU: two calls whose work overlaps on the GPU (different streams, or
// different host threads) race on it. Each call rewrites every byte it later
// reads, so nothing in the array has to start at zero and leftovers of the
// previous call are never used.
// ---------------------------------------------------------------------------

#include <cuda.h>

#include <mutex>

namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;   // 32 MiB per GPU
constexpr int kMaxDevices = 64;
}  // namespace

static __device__ __align__(256) unsigned char g_bsa_noalloc_scratch[kNoAllocScratchBytes];

namespace {

// The scratch array's device address is a property of the CUDA context that
// loaded this library's module: a new primary context (after cudaDeviceReset,
// for instance) loads the module again, and the array may then sit elsewhere.
// So the address is cached per device together with the id of the context it
// was looked up in (cuCtxGetId: unique for the life of the process, never
// reused), and looked up again, with that device current, whenever the
// current context is another one. Failed lookups are not cached.
struct ScratchSlot {
    std::mutex mu;
    unsigned long long ctx_id = 0;   // 0: nothing cached
    void *ptr = nullptr;
};
ScratchSlot g_scratch[kMaxDevices];

typedef CUresult (*PFN_ctx_get_current)(CUcontext *);
typedef CUresult (*PFN_ctx_get_id)(CUcontext, unsigned long long *);

bool driver_fn(const char *name, void **fn) {
    cudaDriverEntryPointQueryResult q;
    return cudaGetDriverEntryPoint(name, fn, cudaEnableDefault, &q) == cudaSuccess &&
           q == cudaDriverEntryPointSuccess && *fn != nullptr;
}

// Id of the calling thread's current context, or 0 if there is none (yet).
cudaError_t current_ctx_id(unsigned long long *id) {
    static PFN_ctx_get_current get_current = nullptr;
    static PFN_ctx_get_id get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *f = nullptr;
        if (driver_fn("cuCtxGetCurrent", &f)) get_current = reinterpret_cast<PFN_ctx_get_current>(f);
        f = nullptr;
        if (driver_fn("cuCtxGetId", &f)) get_id = reinterpret_cast<PFN_ctx_get_id>(f);
    });
    if (!get_current || !get_id) return cudaErrorNotSupported;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    *id = 0;
    if (ctx && get_id(ctx, id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
    return cudaSuccess;
}

// Device address of the scratch array in the current device's current context.
// In host code the array's name only stands in for it, so the address is
// looked up with cudaGetSymbolAddress, once per device and context, on the
// first call made there.
cudaError_t noalloc_scratch(void **out) {
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    ScratchSlot &slot = g_scratch[dev];
    std::lock_guard<std::mutex> lock(slot.mu);
    unsigned long long id = 0;
    if ((e = current_ctx_id(&id)) != cudaSuccess) return e;
    if (id != 0 && id == slot.ctx_id && slot.ptr) {
        *out = slot.ptr;
        return cudaSuccess;
    }
    void *p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_bsa_noalloc_scratch)) != cudaSuccess) return e;   // not cached
    if (!p) return cudaErrorInvalidSymbol;
    if ((e = current_ctx_id(&id)) != cudaSuccess) return e;   // the lookup may have created the context
    slot.ctx_id = id;
    slot.ptr = p;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" bsa_status bsa_forward_noalloc(const bsa_config *cfg, const void *q, const void *k, const void *v,
                                          const float *gates, void *out, int32_t *sel_idx_out,
                                          uint32_t *status_word, cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!q || !k || !v || !gates || !out) return BSA_ERR_INVALID_ARG;
    const WorkspaceLayout L = layout_of(p);
    if (L.base > kNoAllocScratchBytes) return BSA_ERR_WORKSPACE;    // problem too large for the fixed scratch
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gates) || !aligned16(out) ||
        !aligned16(sel_idx_out) || ((uintptr_t)status_word & 3u))
        return BSA_ERR_ALIGNMENT;
    void *scratch = nullptr;
    if (noalloc_scratch(&scratch) != cudaSuccess) return BSA_ERR_CUDA;
    char *ws = static_cast<char *>(scratch);
    float *qbar = reinterpret_cast<float *>(ws + L.qbar);
    float *kbar = reinterpret_cast<float *>(ws + L.kbar);
    float *vbar = reinterpret_cast<float *>(ws + L.vbar);
    float *ocg = reinterpret_cast<float *>(ws + L.o_cg);
    int32_t *idx = sel_idx_out ? sel_idx_out : reinterpret_cast<int32_t *>(ws + L.idx);
    cudaError_t e = bsa::launch_pool(p, q, k, v, qbar, kbar, vbar, stream);
    if (e == cudaSuccess) e = launch_compress(p, qbar, kbar, vbar, ocg, idx, status_word, nullptr, stream);
    if (e == cudaSuccess) e = launch_fine(p, q, k, v, gates, ocg, idx, out, status_word, stream);
    return from_cuda(e);
}

// ---------------------------------------------------------------------------
// Test hook (include/bsa_testing.h): the tensor-core fine-attention kernel
// with one V copy withheld, so that a bounded wait expires on purpose.
// ---------------------------------------------------------------------------
extern "C" bsa_status bsa_testing_fine_attention_withhold(const bsa_config *cfg, const void *q, const void *k,
                                                           const void *v, const float *gates,
                                                           const float *o_cg_block, const int32_t *sel_idx,
                                                           void *out, uint32_t *status_word,
                                                           int64_t withhold_v_step, cudaStream_t stream) {
    Problem p;
    bsa_status st = make_problem(cfg, &p);
    if (st != BSA_OK) return st;
    if (!q || !k || !v || !gates || !o_cg_block || !sel_idx || !out || !status_word) return BSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(gates) || !aligned16(o_cg_block) ||
        !aligned16(sel_idx) || !aligned16(out) || ((uintptr_t)status_word & 3u))
        return BSA_ERR_ALIGNMENT;
    if (withhold_v_step < 0) return BSA_ERR_INVALID_ARG;
    p.withhold_v_step = withhold_v_step;
    return from_cuda(bsa::launch_attend_tc(p, q, k, v, gates, o_cg_block, sel_idx, out, status_word, stream));
}

// Test hook (include/bsa_testing.h): the softmax's two exp2 routes, elementwise.
extern "C" bsa_status bsa_testing_exp2(const float *x, float *y, int64_t n, int32_t poly, cudaStream_t stream) {
    if (!x || !y || n < 0) return BSA_ERR_INVALID_ARG;
    if (((uintptr_t)x & 3u) || ((uintptr_t)y & 3u)) return BSA_ERR_ALIGNMENT;
    if (n == 0) return BSA_OK;
    return from_cuda(bsa::launch_exp2_eval(x, y, n, poly, stream));
}

// Test hook (include/bsa_testing.h): tcgen05.mma issue and execution rate of an m x n tile.
extern "C" bsa_status bsa_testing_mma_rate(int32_t m, int32_t n, int32_t warps, int64_t *cycles,
                                           cudaStream_t stream) {
    if (!cycles || (m != 64 && m != 128) || (n != 64 && n != 128 && n != 256) ||
        (warps != 1 && warps != 2 && warps != 4))
        return BSA_ERR_INVALID_ARG;
    if ((uintptr_t)cycles & 7u) return BSA_ERR_ALIGNMENT;
    return from_cuda(bsa::launch_mma_rate(m, n, warps, reinterpret_cast<long long *>(cycles), stream));
}

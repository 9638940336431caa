/*
 * bsa.h — C ABI of the B200 (sm_100a) forward pass of mesh-aligned
 * block-sparse attention (BSA) over a HEALPix NESTED token sequence.
 *
 * The operation is the one the MOSAIC note defines ("(Sparse) Attention to
 * the Details", papernotes.org ICML 2026 page, section "Mesh-aligned
 * Block-Sparse Attention (BSA)"): the N tokens of one (batch, head) slab are
 * cut into m = N / block_size contiguous blocks, each block is mean-pooled
 * into q̄, k̄, v̄; (a) a compressed branch computes softmax_j(q̄_i·k̄_j·s)
 * block to block and gives every token of block i the vector
 * o_CG_i = Σ_j ā_ij v̄_j; (b) each query block keeps the top-n key blocks by
 * compressed logit and every one of its tokens attends at full resolution to
 * the tokens of those n blocks; (c) every token attends to the tokens of the
 * block-aligned window of blocks max(0,i-w) .. min(m-1,i+w); finally
 * o = g_CG·o_CG + g_FG·o_FG + g_L·o_L with per-token gates.
 *
 * Conventions shared by every call
 *  - Layouts are row-major and contiguous:
 *      q, k, v, out   [batch][heads][n_tokens][head_dim]   element type = cfg->dtype
 *      gates          [batch][heads][n_tokens][3]          float, order (CG, FG, L)
 *      qbar/kbar/vbar [batch][heads][m][head_dim]          float
 *      o_cg_block     [batch][heads][m][head_dim]          float
 *      sel_idx        [batch][heads][m][top_n]             int32, block indices in [0, m),
 *                     ordered by logit descending, equal logits by lower index.
 *  - Every pointer is a DEVICE pointer owned by the caller and must be 16-byte
 *    aligned. The library allocates nothing, frees nothing and never
 *    synchronises (except bsa_check_status). All calls are asynchronous on
 *    `stream` (0 = the legacy default stream) of the current device.
 *  - Errors found on the host return before anything is launched. A launch
 *    failure returns BSA_ERR_CUDA. Errors found by a kernel (an index out of
 *    range in a caller-supplied sel_idx, a bounded wait that expired) are
 *    OR-ed into a 32-bit device status word; bsa_check_status reads it.
 *  - Supported shapes: (dtype, block_size, head_dim) in
 *      {(BSA_F32, 16, 32), (BSA_F32, 64, 64), (BSA_BF16, 64, 64)}
 *    with 1 <= top_n <= min(m, 64) and window_blocks >= 0. bf16 inputs use
 *    bf16 tensor-core products with fp32 accumulation; the compressed
 *    branch and the top-n decision are fp32-accurate (fp32 on the CUDA
 *    cores, or, for head_dim 64 and top_n 16 or 32, three-pass tf32 products
 *    on the tensor cores).
 */
#ifndef BSA_H
#define BSA_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BSA_OK = 0,
    BSA_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, N % block_size != 0, n > m, ... */
    BSA_ERR_UNSUPPORTED = 2,  /* valid problem outside the compiled (dtype, block, head_dim, top_n) set */
    BSA_ERR_ALIGNMENT = 3,    /* a pointer is not 16-byte aligned */
    BSA_ERR_CUDA = 4,         /* a CUDA runtime call or kernel launch failed */
    BSA_ERR_TIMEOUT = 5,      /* a kernel's bounded wait expired (reported via the status word) */
    BSA_ERR_WORKSPACE = 6,    /* workspace missing or smaller than bsa_workspace_size() */
    BSA_ERR_INDEX = 7         /* a kernel met a block index outside [0, m) (via the status word) */
} bsa_status;

typedef enum { BSA_F32 = 0, BSA_BF16 = 1 } bsa_dtype;

typedef struct {
    int32_t batch;          /* B >= 1 */
    int32_t heads;          /* H >= 1 */
    int32_t n_tokens;       /* N, NESTED order; N % block_size == 0 */
    int32_t head_dim;       /* d */
    int32_t block_size;     /* tokens per block (4^L for one parent pixel) */
    int32_t top_n;          /* key blocks selected per query block, 1 <= n <= m */
    int32_t window_blocks;  /* w: local window = blocks i-w .. i+w, clamped */
    int32_t dtype;          /* bsa_dtype of q, k, v, out */
    float scale;            /* logit scale s; 0 means 1/sqrt(head_dim) */
} bsa_config;

/*
 * Step "pooling φ" of the BSA section: block means
 *   qbar[b][h][j][c] = (1/block_size) Σ_{t in block j} q[b][h][t][c]   (same for k, v)
 * computed with fp32 accumulation from 16-byte vector loads.
 */
BSA_API bsa_status bsa_pool(const bsa_config *cfg, const void *q, const void *k, const void *v,
                    float *qbar, float *kbar, float *vbar, cudaStream_t stream);

/*
 * Branch (a) and the top-n choice of branch (b) of the BSA section, with
 * fp32-accurate arithmetic:
 *   z_ij = s·q̄_i·k̄_j,  o_cg_block[i] = Σ_j softmax_j(z_ij) v̄_j,
 *   sel_idx[i] = the top_n blocks j by (z_ij descending, j ascending).
 * The m×m logit matrix is never written to memory. For head_dim 64 and
 * top_n 16 or 32 the products run on the tensor cores as three tf32 products each
 * (operands split into tf32 high and low parts); other shapes use fp32 on the
 * CUDA cores. The tensor-core kernel bounds every internal wait (2 s); should
 * one expire, the affected rows get -1 as their block indices (which
 * bsa_fine_attention then flags as BSA_ERR_INDEX).
 */
BSA_API bsa_status bsa_compress_select(const bsa_config *cfg, const float *qbar, const float *kbar,
                               const float *vbar, float *o_cg_block, int32_t *sel_idx,
                               cudaStream_t stream);

/*
 * The same computation with a caller-owned device workspace (the one
 * bsa_forward takes: >= bsa_workspace_size bytes, 256-byte aligned). On the
 * tensor-core path it first writes the tf32 split of q̄, k̄, v̄ into the
 * workspace once per slab, so that the compressed kernel need not split every
 * key tile again in every CTA; results are identical to bsa_compress_select.
 * Only the split region of the workspace is written (it is the region after
 * the block indices); BSA_ERR_WORKSPACE if the workspace is missing or small.
 */
BSA_API bsa_status bsa_compress_select_ws(const bsa_config *cfg, const float *qbar, const float *kbar,
                                  const float *vbar, float *o_cg_block, int32_t *sel_idx, void *workspace,
                                  size_t workspace_bytes, cudaStream_t stream);

/*
 * Branches (b) and (c) and the gated combine of the BSA section, given the
 * block-level compressed output and the selected block indices:
 *   out_t = g_CG,t·o_cg_block[i(t)] + g_FG,t·o_FG,t + g_L,t·o_L,t
 * with o_FG,t softmax attention of q_t over the tokens of sel_idx[i(t)][0..n)
 * and o_L,t over the tokens of blocks max(0,i-w)..min(m-1,i+w).
 * sel_idx entries outside [0, m) are skipped and flagged BSA_ERR_INDEX in
 * *status_word (nullable, device uint32, OR-ed, never cleared here).
 */
BSA_API bsa_status bsa_fine_attention(const bsa_config *cfg, const void *q, const void *k, const void *v,
                              const float *gates, const float *o_cg_block, const int32_t *sel_idx,
                              void *out, uint32_t *status_word, cudaStream_t stream);

/* Bytes of device workspace bsa_forward needs for cfg (status word, pooled
 * tensors, o_cg_block, block indices, and, on the tensor-core compressed path,
 * the tf32 split of the pooled tensors). */
BSA_API bsa_status bsa_workspace_size(const bsa_config *cfg, size_t *bytes);

/*
 * The whole forward pass: bsa_pool -> bsa_compress_select -> bsa_fine_attention,
 * three kernels on `stream`. `workspace` (device, >= bsa_workspace_size bytes,
 * 256-byte aligned) holds the intermediates; its first 4 bytes are the status
 * word, which must be zero before the first call (e.g. allocate it zeroed)
 * and is reset by bsa_check_status. sel_idx_out (nullable) receives a copy of
 * the selected block indices [B][H][m][top_n].
 */
BSA_API bsa_status bsa_forward(const bsa_config *cfg, const void *q, const void *k, const void *v,
                       const float *gates, void *out, int32_t *sel_idx_out,
                       void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Synchronises `stream`, reads the device status word at `status_word`
 * (the start of a bsa_forward workspace, or the word given to
 * bsa_fine_attention), resets it to zero and returns BSA_OK, BSA_ERR_TIMEOUT
 * or BSA_ERR_INDEX (BSA_ERR_CUDA if the copy itself fails).
 */
BSA_API bsa_status bsa_check_status(const void *status_word, cudaStream_t stream);

/*
 * bsa_forward whose fine-attention epilogue also stores every output row, at
 * the same offset as in `out`, into n_mirrors further buffers (0..7; a host
 * array of device pointers, 16-byte aligned, none equal to out): the
 * all-gather of a forward sharded by (batch, head) slab over the GPUs of one
 * node, done by the kernel's own stores as each tile finishes. In that use
 * every rank passes, as `out` and mirrors, its slab range within its own and
 * its peers' full output buffers (peer memory mapped over NVLink, e.g.
 * symmetric memory); the caller synchronises the ranks afterwards (a system
 * barrier) before reading peers' rows. bf16 only (the tensor-core kernel);
 * otherwise as bsa_forward. Not a step of the method: its distribution.
 */
BSA_API bsa_status bsa_forward_mirrored(const bsa_config *cfg, const void *q, const void *k, const void *v,
                                        const float *gates, void *out, void *const *mirrors, int32_t n_mirrors,
                                        int32_t *sel_idx_out, void *workspace, size_t workspace_bytes,
                                        cudaStream_t stream);

/*
 * Lat-lon -> HEALPix cross-attention interpolation, the step before BSA in
 * the MOSAIC note's pipeline ("overall framework", step (1), and the HEALPix
 * paragraph): every HEALPix target pixel i attends to its neighbouring source
 * points j of a latitude-longitude grid, with the relative position p_ij as
 * the query and the source features as keys and values,
 *   o_i = Σ_{j in N_i} softmax_j((W_q p_ij)·k_j · s) v_j.
 *
 * bsa_latlon_healpix_plan: for the 12·nside² NESTED pixels (nside a power of
 * two) over a grid of nlat rows (+90 .. -90 degrees, poles included) and nlon
 * columns (0 degrees eastwards, source index row*nlon + col): N_i, the 4 x 4
 * grid points around the pixel centre (rows r0..r0+3 with r0 = floor((90 -
 * lat)/dlat) - 1 clamped to [0, nlat-4]; columns c0-1..c0+2 wrapping in
 * longitude, c0 = floor(lon/dlon)), written to nbr [npix][16] int32, and
 * p_ij = (x_j - x_i)/dlat_rad (unit vectors, grid step in radians) to rel
 * [npix][16][3] float. Device buffers, 16-byte aligned.
 *
 * bsa_latlon_to_healpix: the attention over such a plan for `batch`
 * independent feature sets: k_src, v_src [batch][n_src][head_dim] and out
 * [batch][n_tgt][head_dim] in `dtype` (bf16 or fp32), wq [head_dim][3]
 * float (the query map), scale 0 = 1/sqrt(head_dim); head_dim 32, 64 or 128.
 * fp32 arithmetic. The logits are formed as p_ij·(W_qᵀ k_j), the same value
 * as (W_q p_ij)·k_j: each source key is reduced once to 3 floats, kept in
 * `workspace` (device, 16-byte aligned, >= bsa_latlon_workspace_size bytes;
 * BSA_ERR_WORKSPACE otherwise). Neighbour indices outside [0, n_src) are
 * replaced by 0 and flagged BSA_ERR_INDEX in *status_word (nullable).
 */
BSA_API bsa_status bsa_latlon_healpix_plan(int64_t nside, int64_t nlat, int64_t nlon, int32_t *nbr, float *rel,
                                           cudaStream_t stream);
BSA_API bsa_status bsa_latlon_workspace_size(int64_t batch, int64_t n_src, size_t *bytes);
BSA_API bsa_status bsa_latlon_to_healpix(int64_t batch, int64_t n_tgt, int64_t n_src, int64_t head_dim,
                                         int32_t dtype, float scale, const int32_t *nbr, const float *rel,
                                         const float *wq, const void *k_src, const void *v_src, void *out,
                                         void *workspace, size_t workspace_bytes, uint32_t *status_word,
                                         cudaStream_t stream);

/*
 * Token layouts other than HEALPix NESTED. The note's ablation "BSA but not
 * HEALPix (lat-lon block)" takes the blocks from a latitude-longitude grid;
 * BSA itself needs each block contiguous, so such a layout is brought into
 * block-contiguous order before the forward and back after it:
 *   dst[s][t][:] = src[s][perm[t]][:]   for every slab s < slabs, t < n_tokens
 * Rows are row_bytes long (head_dim x element size, or 3 x 4 for gates; a
 * multiple of 4), src and dst distinct device buffers of slabs*n_tokens rows
 * (16-byte aligned when row_bytes is a multiple of 16, else 4-byte aligned),
 * perm a device int32 [n_tokens] shared by all slabs (a
 * permutation: entries outside [0, n_tokens) are skipped and flagged
 * BSA_ERR_INDEX in *status_word, nullable). The inverse move uses the
 * inverse permutation.
 */
BSA_API bsa_status bsa_permute_tokens(int64_t slabs, int64_t n_tokens, int64_t row_bytes, const int32_t *perm,
                                      const void *src, void *dst, uint32_t *status_word, cudaStream_t stream);

/*
 * Training. The MOSAIC note trains its model through BSA ("loss function /
 * training strategy" sections: autoregressive training on ERA5), so the
 * library provides the gradient of the forward above. The top-n choice is a
 * discrete decision and carries no gradient: the backward holds the selected
 * blocks fixed, and the compressed branch carries the gradient to the pooled
 * keys and values it attends over. bf16 with block_size 64 and head_dim 64
 * only (BSA_ERR_UNSUPPORTED otherwise).
 *
 * bsa_forward_train: bsa_forward plus the tensors bsa_backward needs, all
 * caller-owned device buffers (16-byte aligned):
 *   sel_idx    [B][H][m][top_n] int32   selected blocks (as bsa_forward's sel_idx_out)
 *   o_cg_block [B][H][m][d]     float   compressed-branch output per query block
 *   lse_cg     [B][H][m]        float   ln Σ_j exp(z_ij) of each compressed row
 *   o_fg, o_l  [B][H][N][d]     dtype   selection and local branch outputs (before the gates)
 *   lse_fine   [B][H][N][2]     float   ln Σ_u exp(s·q_t·k_u) of each token over its
 *                                       selected (index 0) and local (index 1) keys
 * workspace as for bsa_forward (bsa_workspace_size bytes, status word first).
 */
BSA_API bsa_status bsa_forward_train(const bsa_config *cfg, const void *q, const void *k, const void *v,
                                     const float *gates, void *out, int32_t *sel_idx, float *o_cg_block,
                                     float *lse_cg, void *o_fg, void *o_l, float *lse_fine, void *workspace,
                                     size_t workspace_bytes, cudaStream_t stream);

/* Bytes of device workspace bsa_backward needs for cfg. */
BSA_API bsa_status bsa_backward_workspace_size(const bsa_config *cfg, size_t *bytes);

/*
 * Gradients of L with respect to q, k, v and the gates, given dout = dL/dout
 * ([B][H][N][d], dtype) and the tensors bsa_forward_train saved:
 *   dq, dk, dv [B][H][N][d] dtype,  dgates [B][H][N][3] float (CG, FG, L).
 * Chain rule through the combine (dgates_t = dout_t·(o_CG, o_FG, o_L)), the
 * selection and local softmax rows, the compressed branch (block level) and
 * the mean pooling (each token gets 1/block_size of its block's pooled
 * gradient). Runs on `stream` with `workspace` (device, >= bsa_backward_workspace_size
 * bytes, 256-byte aligned; its first 4 bytes are a status word, as in
 * bsa_forward, read by bsa_check_status). Accumulates in fp32; dq, dk, dv
 * are rounded to dtype once at the end. Block indices outside [0, m) in
 * sel_idx are skipped and flagged BSA_ERR_INDEX in the status word.
 */
BSA_API bsa_status bsa_backward(const bsa_config *cfg, const void *q, const void *k, const void *v,
                                const float *gates, const void *dout, const int32_t *sel_idx,
                                const float *o_cg_block, const float *lse_cg, const void *o_fg, const void *o_l,
                                const float *lse_fine, void *dq, void *dk, void *dv, float *dgates,
                                void *workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Allocation-free variant of bsa_forward (the MOSAIC note has no counterpart:
 * this is a deployment convenience, not a step of the method).
 *
 * For callers that cannot allocate device memory when they run BSA (code in
 * a host callback or an allocator hook, plugins whose host framework owns all
 * device allocations, request paths that must not touch the allocator). It
 * computes what bsa_forward computes (bit for bit), but the intermediates
 * live in a fixed 32 MiB array of device memory owned by the library instead
 * of a caller workspace, and the compressed branch splits its operands inside
 * every CTA, as bsa_compress_select does; the caller still passes q, k, v,
 * gates and out (and the
 * optional sel_idx_out / status_word, same meaning as in bsa_forward and
 * bsa_fine_attention; status_word may be NULL).
 *  - Returns BSA_ERR_WORKSPACE when the intermediates (status word, pooled
 *    tensors, o_cg_block, block indices: bsa_workspace_size without the
 *    compressed kernel's split images) exceed 32 MiB (e.g. Nside 64 with
 *    batch 4 x 8 heads fits; Nside 128 with 2 x 16 does not).
 *  - Never calls cudaMalloc, cudaFree or any allocating routine.
 *  - The array exists on every GPU that loads the library until the process
 *    exits. The first call on each device looks up its device address (with
 *    that device current); make that first call before any stream capture.
 *    The address is remembered per device and CUDA context: a call made in a
 *    new context of the device (e.g. after cudaDeviceReset) looks it up
 *    again, and a lookup that fails is retried by the next call.
 *  - All calls on a GPU share the array: calls that overlap on the GPU
 *    (other streams, other host threads) race and must be serialised by the
 *    caller. Each call rewrites everything it reads, so no part of the array
 *    needs to start at zero.
 */
BSA_API bsa_status bsa_forward_noalloc(const bsa_config *cfg, const void *q, const void *k, const void *v,
                                       const float *gates, void *out, int32_t *sel_idx_out,
                                       uint32_t *status_word, cudaStream_t stream);

/* Static, human-readable name of a status code. */
BSA_API const char *bsa_status_string(bsa_status status);

#ifdef __cplusplus
}
#endif

#endif /* BSA_H */

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
 *    cores, or, for head_dim 64 and top_n 16, three-pass tf32 products on
 *    the tensor cores).
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
 * top_n 16 the products run on the tensor cores as three tf32 products each
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

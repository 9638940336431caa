// Internal declarations shared by the BSA CUDA translation units.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "bsa.h"

namespace bsa {

// Status-word bits written by kernels (atomicOr).
constexpr uint32_t kStatusTimeout = 1u << 0;
constexpr uint32_t kStatusBadIndex = 1u << 1;

// Largest top_n the compressed/select kernel keeps per query block.
constexpr int kMaxTopN = 64;

struct Problem {
    int64_t batch, heads, n_tokens, head_dim, block_size, top_n, window;
    int64_t m;        // blocks per slab
    int64_t slabs;    // batch * heads
    bsa_dtype dtype;
    float scale;      // logit scale s
    // Test hook: when >= 0 the tensor-core kernel's first pipeline skips the V
    // copy of this step, so that the wait for it expires (bounded-wait test).
    int64_t withhold_v_step = -1;
};

// Launchers (return cudaGetLastError()).
cudaError_t launch_pool(const Problem &p, const void *q, const void *k, const void *v,
                        float *qbar, float *kbar, float *vbar, cudaStream_t stream);
// lse (nullable, [slabs*m] float): training output, the natural-log log-sum-exp of each
// row's scaled logits.
cudaError_t launch_compress_select(const Problem &p, const float *qbar, const float *kbar,
                                   const float *vbar, float *o_cg, int32_t *idx,
                                   cudaStream_t stream, float *lse = nullptr);
// tcgen05 three-pass tf32 path for (head_dim 64, top_n 16 or 32). Returns
// cudaErrorNotSupported when it cannot take the problem. status: nullable.
// images: nullable device scratch of compress_tc_workspace_bytes(p) bytes
// (16-byte aligned); with it the tf32 split is done once per slab.
bool compress_tc_supported(const Problem &p);
size_t compress_tc_workspace_bytes(const Problem &p);
cudaError_t launch_compress_tc(const Problem &p, const float *qbar, const float *kbar, const float *vbar,
                               float *o_cg, int32_t *idx, uint32_t *status, void *images, cudaStream_t stream,
                               float *lse = nullptr);
cudaError_t launch_attend_simt(const Problem &p, const void *q, const void *k, const void *v,
                               const float *gates, const float *o_cg, const int32_t *idx,
                               void *out, uint32_t *status, cudaStream_t stream);
// tcgen05/TMA path for (bf16, block 64, d 64), the only kernel for bf16 fine
// attention. Returns cudaErrorNotSupported for shapes it does not take.
// o_fg, o_l ([slabs*N][64] bf16) and lse ([slabs*N][2] float): optional training outputs
// (all null or all set): normalised branch outputs and per-branch row log-sum-exp.
cudaError_t launch_attend_tc(const Problem &p, const void *q, const void *k, const void *v,
                             const float *gates, const float *o_cg, const int32_t *idx,
                             void *out, uint32_t *status, cudaStream_t stream, void *o_fg = nullptr,
                             void *o_l = nullptr, float *lse = nullptr, void *const *mirrors = nullptr,
                             int n_mirrors = 0);

// dst[s][t] = src[s][perm[t]] (rows of row_bytes, a multiple of 16); perm entries
// outside [0, n_tokens) are skipped and flagged in *status (nullable).
cudaError_t launch_permute_rows(const void *src, void *dst, const int32_t *perm, int64_t slabs, int64_t n_tokens,
                                int64_t row_bytes, uint32_t *status, cudaStream_t stream);

// Lat-lon -> HEALPix interpolation: the plan (16 neighbours and relative positions of
// every NESTED pixel) and the attention over it.
cudaError_t launch_healpix_plan(int64_t nside, int64_t nlat, int64_t nlon, int32_t *nbr, float *rel,
                                cudaStream_t stream);
cudaError_t launch_interp(int64_t batch, int64_t n_tgt, int64_t n_src, int64_t d, bsa_dtype dtype,
                          const int32_t *nbr, const float *rel, const float *wq, const void *k, const void *v,
                          void *out, float scale, float *kappa, uint32_t *status, cudaStream_t stream);

// Test hook: the fine-attention kernel's exp2 on the FMA pipe (poly != 0) or the exp unit.
cudaError_t launch_exp2_eval(const float *x, float *y, int64_t n, int poly, cudaStream_t stream);
// Test hook: cycles of `warps` threads (one per warp) each issuing 256 back-to-back bf16 tcgen05.mma
// of an m x n tile (K = 16) through completion, into cycles[0..warps) (device); -1 on a timeout.
cudaError_t launch_mma_rate(int m, int n, int warps, long long *cycles, cudaStream_t stream);
int mma_rate_mmas_per_warp();

// ---- backward (training) ------------------------------------------------

// Tensors of one backward pass (bf16, block 64, head_dim 64): the caller's inputs
// and outputs and the regions of the backward workspace.
struct BwdBuffers {
    // inputs
    const void *q, *k, *v, *dout;   // [slabs*N][64] bf16
    const float *gates;             // [slabs*N][3]
    const int32_t *sel_idx;         // [slabs*m][n]
    const float *o_cg, *lse_cg;     // [slabs*m][64], [slabs*m] (training forward)
    const void *o_fg, *o_l;         // [slabs*N][64] bf16 (training forward)
    const float *lse_fine;          // [slabs*N][2]
    // outputs
    void *dq, *dk, *dv;             // [slabs*N][64] bf16
    float *dgates;                  // [slabs*N][3]
    // workspace
    int64_t m_pad;                  // m rounded up to a multiple of 64
    uint32_t *status;
    float *qbar, *kbar, *vbar;      // [slabs*m][64]
    float *dfine;                   // [slabs*N][2]: D of the FG and L rows
    void *docg16, *q16, *k16, *v16; // [slabs*m_pad][64] bf16 (zero rows past m)
    float *dcg, *lse_cg_pad;        // [slabs*m_pad]
    float *dqbar, *dkbar, *dvbar;   // [slabs*m_pad][64]: gradients of q̄, k̄, v̄
    int *count, *offs, *cursor, *list_tmp, *list;   // the inverted selection
};
cudaError_t launch_bwd_prep(const Problem &p, const BwdBuffers &b, cudaStream_t stream);
cudaError_t launch_inverse_index(const Problem &p, const int32_t *idx, int *count, int *offs, int *cursor,
                                 int *list_tmp, int *list, uint32_t *status, cudaStream_t stream);
// Attention backward on the tensor cores: the compressed branch (by key tile, dense
// over the 64-block tiles of q̄, k̄, v̄, dO_CG; dq̄ reduced into b.dqbar) and the two
// fine branches (dk, dv by key tile over each key block's window and the query
// blocks that selected it; then dq by query tile over its selected and window blocks).
cudaError_t launch_attend_bwd_compressed(const Problem &p, const BwdBuffers &b, cudaStream_t stream);
cudaError_t launch_attend_bwd_fine(const Problem &p, const BwdBuffers &b, cudaStream_t stream);

// ---- small device helpers ------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

}  // namespace bsa

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
cudaError_t launch_compress_select(const Problem &p, const float *qbar, const float *kbar,
                                   const float *vbar, float *o_cg, int32_t *idx,
                                   cudaStream_t stream);
// tcgen05 three-pass tf32 path for (head_dim 64, top_n 16). Returns
// cudaErrorNotSupported when it cannot take the problem. status: nullable.
// images: nullable device scratch of compress_tc_workspace_bytes(p) bytes
// (16-byte aligned); with it the tf32 split is done once per slab.
bool compress_tc_supported(const Problem &p);
size_t compress_tc_workspace_bytes(const Problem &p);
cudaError_t launch_compress_tc(const Problem &p, const float *qbar, const float *kbar, const float *vbar,
                               float *o_cg, int32_t *idx, uint32_t *status, void *images, cudaStream_t stream);
cudaError_t launch_attend_simt(const Problem &p, const void *q, const void *k, const void *v,
                               const float *gates, const float *o_cg, const int32_t *idx,
                               void *out, uint32_t *status, cudaStream_t stream);
// tcgen05/TMA path for (bf16, block 64, d 64), the only kernel for bf16 fine
// attention. Returns cudaErrorNotSupported for shapes it does not take.
cudaError_t launch_attend_tc(const Problem &p, const void *q, const void *k, const void *v,
                             const float *gates, const float *o_cg, const int32_t *idx,
                             void *out, uint32_t *status, cudaStream_t stream);

// ---- small device helpers ------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

}  // namespace bsa

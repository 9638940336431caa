// Selection branch (b), local branch (c) and the gated combine of the BSA
// section (MOSAIC note), on the CUDA cores in fp32.
//
// This instantiation serves the fp32 workloads (tcgen05 has no fp32-exact
// product) and any shape the tensor-core kernel does not take. One CTA owns
// one query block of one slab: BK query rows x TPR threads per row, each
// thread holding D/TPR columns of its row. Key/value blocks are staged in
// shared memory one at a time; each branch runs its own online softmax.
#include <math_constants.h>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int TPR = 4;   // threads per query row

template <typename T, int BK, int D>
__device__ __forceinline__ void stage_block(float *Ks, float *Vs, const T *k, const T *v, int64_t blk) {
    const T *kb = k + blk * (int64_t)(BK * D);
    const T *vb = v + blk * (int64_t)(BK * D);
    for (int e = threadIdx.x; e < BK * D; e += blockDim.x) {
        Ks[e] = to_f32(kb[e]);
        Vs[e] = to_f32(vb[e]);
    }
}

// One online-softmax step over the BK keys staged in Ks/Vs.
template <int BK, int D>
__device__ __forceinline__ void attend_block(const float *Ks, const float *Vs, const float *qs,
                                             int part, float &mrun, float &lrun, float *o) {
    constexpr int DS = D / TPR;
    float sc[BK];
    float mx = -CUDART_INF_F;
#pragma unroll
    for (int u = 0; u < BK; ++u) {
        float d = 0.f;
#pragma unroll
        for (int c = 0; c < DS; ++c) d = fmaf(qs[c], Ks[u * D + part * DS + c], d);
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        d += __shfl_xor_sync(0xffffffffu, d, 2);
        sc[u] = d;
        mx = fmaxf(mx, d);
    }
    const float mnew = fmaxf(mrun, mx);
    const float alpha = exp2f(mrun - mnew);
    float ls = 0.f;
#pragma unroll
    for (int c = 0; c < DS; ++c) o[c] *= alpha;
#pragma unroll
    for (int u = 0; u < BK; ++u) {
        const float p = exp2f(sc[u] - mnew);
        ls += p;
#pragma unroll
        for (int c = 0; c < DS; ++c) o[c] = fmaf(p, Vs[u * D + part * DS + c], o[c]);
    }
    lrun = lrun * alpha + ls;
    mrun = mnew;
}

template <typename T, int BK, int D>
__global__ void __launch_bounds__(BK * TPR)
attend_simt_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
                   const float *__restrict__ gates, const float *__restrict__ o_cg,
                   const int32_t *__restrict__ idx, T *__restrict__ out, uint32_t *status,
                   int m, int n, int w, float scale_log2) {
    constexpr int DS = D / TPR;
    __shared__ float Ks[BK * D];
    __shared__ float Vs[BK * D];
    const int row = threadIdx.x / TPR, part = threadIdx.x % TPR;
    const int i = blockIdx.x;                       // query block
    const int64_t slab = blockIdx.y;
    const int64_t ntok = (int64_t)m * BK;
    const T *qs_ = q + slab * ntok * D;
    const T *ks_ = k + slab * ntok * D;
    const T *vs_ = v + slab * ntok * D;
    const int64_t t = (int64_t)i * BK + row;       // token within the slab

    float qreg[DS];
#pragma unroll
    for (int c = 0; c < DS; ++c) qreg[c] = to_f32(qs_[t * D + part * DS + c]) * scale_log2;

    // (b) selection branch over the n chosen blocks
    float mf = -CUDART_INF_F, lf = 0.f, of[DS];
#pragma unroll
    for (int c = 0; c < DS; ++c) of[c] = 0.f;
    const int32_t *sel = idx + (slab * m + i) * (int64_t)n;
    for (int s = 0; s < n; ++s) {
        const int j = sel[s];
        if (j < 0 || j >= m) {                       // uniform over the CTA
            if (threadIdx.x == 0 && status) atomicOr(status, kStatusBadIndex);
            continue;
        }
        __syncthreads();
        stage_block<T, BK, D>(Ks, Vs, ks_, vs_, j);
        __syncthreads();
        attend_block<BK, D>(Ks, Vs, qreg, part, mf, lf, of);
    }
    // (c) local branch over the clamped window
    float ml = -CUDART_INF_F, ll = 0.f, ol[DS];
#pragma unroll
    for (int c = 0; c < DS; ++c) ol[c] = 0.f;
    const int lo = i - w < 0 ? 0 : i - w;
    const int hi = i + w > m - 1 ? m - 1 : i + w;
    for (int j = lo; j <= hi; ++j) {
        __syncthreads();
        stage_block<T, BK, D>(Ks, Vs, ks_, vs_, j);
        __syncthreads();
        attend_block<BK, D>(Ks, Vs, qreg, part, ml, ll, ol);
    }
    // gated combine
    const float *g = gates + (slab * ntok + t) * 3;
    const float g_cg = g[0], g_fg = g[1], g_l = g[2];
    const float inv_f = lf > 0.f ? 1.0f / lf : 0.f;
    const float inv_l = 1.0f / ll;
    const float *cg = o_cg + (slab * m + i) * (int64_t)D + part * DS;
    T *dst = out + (slab * ntok + t) * D + part * DS;
#pragma unroll
    for (int c = 0; c < DS; ++c)
        dst[c] = from_f32<T>(g_cg * cg[c] + g_fg * (of[c] * inv_f) + g_l * (ol[c] * inv_l));
}

template <typename T, int BK, int D>
cudaError_t launch(const Problem &p, const void *q, const void *k, const void *v, const float *gates,
                   const float *ocg, const int32_t *idx, void *out, uint32_t *status, cudaStream_t s) {
    const dim3 grid((unsigned)p.m, (unsigned)p.slabs);
    const float scale_log2 = p.scale * 1.4426950408889634f;
    attend_simt_kernel<T, BK, D><<<grid, BK * TPR, 0, s>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), gates, ocg, idx,
        static_cast<T *>(out), status, (int)p.m, (int)p.top_n, (int)p.window, scale_log2);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attend_simt(const Problem &p, const void *q, const void *k, const void *v,
                               const float *gates, const float *o_cg, const int32_t *idx,
                               void *out, uint32_t *status, cudaStream_t stream) {
    // fp32 workloads only: bf16 fine attention runs on the tensor cores and nowhere else
    if (p.dtype == BSA_F32 && p.block_size == 64 && p.head_dim == 64)
        return launch<float, 64, 64>(p, q, k, v, gates, o_cg, idx, out, status, stream);
    if (p.dtype == BSA_F32 && p.block_size == 16 && p.head_dim == 32)
        return launch<float, 16, 32>(p, q, k, v, gates, o_cg, idx, out, status, stream);
    return cudaErrorNotSupported;
}

}  // namespace bsa

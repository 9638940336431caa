// Pooling φ of the BSA section (MOSAIC note): the mean of each contiguous
// block of `block_size` NESTED tokens, for q, k and v.
//
// HBM-bound: every input byte is read once with 16-byte non-allocating vector
// loads; one warp reduces one (tensor, slab, block) task, which is a single
// contiguous span of block_size*head_dim elements thanks to the NESTED order.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

__device__ __forceinline__ uint4 ld_stream_v4(const void *p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

template <typename T> struct Vec16;
template <> struct Vec16<float> {
    static constexpr int kElems = 4;
    __device__ __forceinline__ static void add(const uint4 &u, float *acc) {
        acc[0] += __uint_as_float(u.x);
        acc[1] += __uint_as_float(u.y);
        acc[2] += __uint_as_float(u.z);
        acc[3] += __uint_as_float(u.w);
    }
};
template <> struct Vec16<__nv_bfloat16> {
    static constexpr int kElems = 8;
    __device__ __forceinline__ static void add(const uint4 &u, float *acc) {
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            acc[2 * i] += __uint_as_float(w[i] << 16);
            acc[2 * i + 1] += __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

template <typename T, int BK, int D>
__global__ void __launch_bounds__(256)
pool_kernel(const T *__restrict__ q, const T *__restrict__ k, const T *__restrict__ v,
            float *__restrict__ qbar, float *__restrict__ kbar, float *__restrict__ vbar,
            int64_t blocks_per_tensor) {
    constexpr int V = Vec16<T>::kElems;        // elements per 16-byte vector
    constexpr int VPR = D / V;                 // vectors per token row
    constexpr int VEC = BK * D / V;            // vectors per block
    static_assert(D % V == 0 && 32 % VPR == 0, "a row must split evenly over the warp");
    static_assert(VEC % 32 == 0, "a block must split evenly over the warp");
    constexpr int IT = VEC / 32;               // vectors per lane
    constexpr int CH = IT < 16 ? IT : 16;      // vectors in flight per lane
    static_assert(IT % CH == 0, "");

    const int lane = threadIdx.x & 31;
    const int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    if (task >= 3 * blocks_per_tensor) return;
    const int which = (int)(task / blocks_per_tensor);
    const int64_t blk = task - which * blocks_per_tensor;
    const T *src = which == 0 ? q : (which == 1 ? k : v);
    float *dst = which == 0 ? qbar : (which == 1 ? kbar : vbar);

    const uint4 *p = reinterpret_cast<const uint4 *>(src + blk * (int64_t)(BK * D));
    float acc[V];
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = 0.f;
#pragma unroll
    for (int base = 0; base < IT; base += CH) {
        uint4 buf[CH];
#pragma unroll
        for (int i = 0; i < CH; ++i) buf[i] = ld_stream_v4(p + lane + 32 * (base + i));
#pragma unroll
        for (int i = 0; i < CH; ++i) Vec16<T>::add(buf[i], acc);
    }
    // lanes with equal (lane % VPR) hold the same columns: reduce over the rest
#pragma unroll
    for (int off = VPR; off < 32; off <<= 1)
#pragma unroll
        for (int e = 0; e < V; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
    if (lane < VPR) {
        const float inv = 1.0f / (float)BK;
        float4 *o = reinterpret_cast<float4 *>(dst + blk * D + lane * V);
#pragma unroll
        for (int e = 0; e < V; e += 4)
            o[e / 4] = make_float4(acc[e] * inv, acc[e + 1] * inv, acc[e + 2] * inv, acc[e + 3] * inv);
    }
}

template <typename T, int BK, int D>
cudaError_t launch(const Problem &p, const void *q, const void *k, const void *v, float *qb,
                   float *kb, float *vb, cudaStream_t s) {
    const int64_t per_tensor = p.slabs * p.m;
    const int64_t warps = 3 * per_tensor;
    const int64_t ctas = (warps + 7) / 8;
    pool_kernel<T, BK, D><<<(unsigned)ctas, 256, 0, s>>>(
        static_cast<const T *>(q), static_cast<const T *>(k), static_cast<const T *>(v), qb, kb, vb,
        per_tensor);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pool(const Problem &p, const void *q, const void *k, const void *v,
                        float *qbar, float *kbar, float *vbar, cudaStream_t stream) {
    if (p.dtype == BSA_BF16 && p.block_size == 64 && p.head_dim == 64)
        return launch<__nv_bfloat16, 64, 64>(p, q, k, v, qbar, kbar, vbar, stream);
    if (p.dtype == BSA_BF16 && p.block_size == 256 && p.head_dim == 64)
        return launch<__nv_bfloat16, 256, 64>(p, q, k, v, qbar, kbar, vbar, stream);
    if (p.dtype == BSA_BF16 && p.block_size == 1024 && p.head_dim == 64)
        return launch<__nv_bfloat16, 1024, 64>(p, q, k, v, qbar, kbar, vbar, stream);
    if (p.dtype == BSA_F32 && p.block_size == 64 && p.head_dim == 64)
        return launch<float, 64, 64>(p, q, k, v, qbar, kbar, vbar, stream);
    if (p.dtype == BSA_F32 && p.block_size == 16 && p.head_dim == 32)
        return launch<float, 16, 32>(p, q, k, v, qbar, kbar, vbar, stream);
    return cudaErrorNotSupported;
}

}  // namespace bsa

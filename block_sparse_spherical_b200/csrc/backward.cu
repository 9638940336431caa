// Backward pass of BSA (training), the CUDA-core parts: everything around the
// two tensor-core attention-backward launches (attend_bwd_tc.cu).
//
// The forward is o_t = g_CG,t·o_CG,i + g_FG,t·o_FG,t + g_L,t·o_L,t (MOSAIC note,
// BSA section); its gradient follows the chain rule through the combine, the
// three branches and the mean pooling, with the top-n selection held fixed (a
// discrete choice without a gradient):
//   bwd_prep_kernel   per query block: dgates_t = dout_t·(o_CG,i, o_FG,t, o_L,t);
//                     the rows' D terms of the two fine branches,
//                     D_b,t = g_b,t (dout_t·o_b,t); the compressed branch's
//                     incoming gradient dO_CG,i = Σ_t g_CG,t dout_t and its
//                     D_i = dO_CG,i·o_CG,i; bf16 copies of q̄, k̄, v̄ and dO_CG
//                     (rows padded to a multiple of 64 with zeros) for the
//                     tensor-core pass over the compressed branch
//   inv_*_kernel      the selection inverted: for every key block j the query
//                     blocks i whose top-n holds j, ascending (CSR per slab)
#include <math_constants.h>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int HD = 64;

__device__ __forceinline__ float2 ld_bf16x2(const __nv_bfloat16 *p) {
    return __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(p));
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// One CTA (8 warps) per (query block i < m_pad, slab). Lane l of a warp holds
// channels 2l, 2l+1 of a token row.
__global__ void __launch_bounds__(256)
bwd_prep_kernel(const __nv_bfloat16 *__restrict__ dout, const __nv_bfloat16 *__restrict__ o_fg,
                const __nv_bfloat16 *__restrict__ o_l, const float *__restrict__ gates,
                const float *__restrict__ o_cg, const float *__restrict__ lse_cg, const float *__restrict__ qbar,
                const float *__restrict__ kbar, const float *__restrict__ vbar, float *__restrict__ dgates,
                float *__restrict__ dfine, __nv_bfloat16 *__restrict__ docg16, float *__restrict__ dcg,
                float *__restrict__ lse_pad, __nv_bfloat16 *__restrict__ q16, __nv_bfloat16 *__restrict__ k16,
                __nv_bfloat16 *__restrict__ v16, int64_t n_tokens, int m, int m_pad, int block) {
    const int64_t slab = blockIdx.y;
    const int i = blockIdx.x, warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t prow = slab * m_pad + i;         // row of the padded per-block arrays
    __nv_bfloat162 *d16[4] = {reinterpret_cast<__nv_bfloat162 *>(docg16 + prow * HD),
                              reinterpret_cast<__nv_bfloat162 *>(q16 + prow * HD),
                              reinterpret_cast<__nv_bfloat162 *>(k16 + prow * HD),
                              reinterpret_cast<__nv_bfloat162 *>(v16 + prow * HD)};
    if (i >= m) {                                 // padding rows: no keys, no queries
        if (warp < 4) d16[warp][lane] = __floats2bfloat162_rn(0.f, 0.f);
        if (threadIdx.x == 0) {
            dcg[prow] = 0.f;
            lse_pad[prow] = CUDART_INF_F;         // exp(s - inf) = 0: the row takes no part
        }
        return;
    }
    const int64_t brow = slab * m + i;            // row of the unpadded per-block arrays
    const float2 cg = *reinterpret_cast<const float2 *>(o_cg + brow * HD + 2 * lane);
    float a0 = 0.f, a1 = 0.f;                     // this warp's share of dO_CG (channels 2l, 2l+1)
    for (int r = warp; r < block; r += 8) {
        const int64_t t = slab * n_tokens + (int64_t)i * block + r;
        const float2 y = ld_bf16x2(dout + t * HD + 2 * lane);
        const float2 f = ld_bf16x2(o_fg + t * HD + 2 * lane);
        const float2 l = ld_bf16x2(o_l + t * HD + 2 * lane);
        const float s0 = warp_sum(y.x * cg.x + y.y * cg.y);
        const float s1 = warp_sum(y.x * f.x + y.y * f.y);
        const float s2 = warp_sum(y.x * l.x + y.y * l.y);
        const float g0 = __ldg(gates + t * 3), g1 = __ldg(gates + t * 3 + 1), g2 = __ldg(gates + t * 3 + 2);
        if (lane == 0) {
            dgates[t * 3] = s0;
            dgates[t * 3 + 1] = s1;
            dgates[t * 3 + 2] = s2;
            dfine[t * 2] = g1 * s1;
            dfine[t * 2 + 1] = g2 * s2;
        }
        a0 = fmaf(g0, y.x, a0);
        a1 = fmaf(g0, y.y, a1);
    }
    __shared__ float2 part[8][32];
    part[warp][lane] = make_float2(a0, a1);
    __syncthreads();
    if (warp == 0) {
        float2 s = part[0][lane];
#pragma unroll
        for (int w = 1; w < 8; ++w) {
            s.x += part[w][lane].x;
            s.y += part[w][lane].y;
        }
        d16[0][lane] = __floats2bfloat162_rn(s.x, s.y);
        const float D = warp_sum(s.x * cg.x + s.y * cg.y);
        if (lane == 0) {
            dcg[prow] = D;
            lse_pad[prow] = __ldg(lse_cg + brow);
        }
    } else if (warp < 4) {
        const float *src = (warp == 1 ? qbar : warp == 2 ? kbar : vbar) + brow * HD + 2 * lane;
        const float2 x = *reinterpret_cast<const float2 *>(src);
        d16[warp][lane] = __floats2bfloat162_rn(x.x, x.y);
    }
}

// ---- selection inverted per slab: CSR (offsets [m+1], query blocks) -------

__global__ void inv_count_kernel(const int32_t *__restrict__ idx, int64_t total, int m, int n,
                                 int *__restrict__ count, uint32_t *status) {
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t slab = e / ((int64_t)m * n);
        const int j = __ldg(idx + e);
        if (j < 0 || j >= m) {
            if (status) atomicOr(status, kStatusBadIndex);
            continue;
        }
        atomicAdd(count + slab * m + j, 1);
    }
}

// One CTA per slab: offs[j] = Σ_{j' < j} count[j'] (offs[m] = total).
__global__ void __launch_bounds__(1024) inv_scan_kernel(const int *__restrict__ count, int *__restrict__ offs, int m) {
    const int64_t slab = blockIdx.x;
    const int *c = count + slab * m;
    int *o = offs + slab * (m + 1);
    __shared__ int warp_tot[32];
    __shared__ int carry;
    if (threadIdx.x == 0) carry = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int base = 0; base < m; base += 1024) {
        const int j = base + threadIdx.x;
        const int x = j < m ? c[j] : 0;
        int incl = x;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int t = warp_tot[lane], ti = t;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, ti, off);
                if (lane >= off) ti += y;
            }
            warp_tot[lane] = ti - t;              // exclusive prefix of the warp totals
        }
        __syncthreads();
        const int excl = carry + warp_tot[warp] + incl - x;
        if (j < m) o[j] = excl;
        __syncthreads();
        if (threadIdx.x == 1023) carry = excl + x;
        __syncthreads();
    }
    if (threadIdx.x == 0) o[m] = carry;
}

__global__ void inv_fill_kernel(const int32_t *__restrict__ idx, int64_t total, int m, int n,
                                const int *__restrict__ offs, int *__restrict__ cursor, int *__restrict__ list) {
    for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t per = (int64_t)m * n, slab = e / per;
        const int i = (int)((e - slab * per) / n);
        const int j = __ldg(idx + e);
        if (j < 0 || j >= m) continue;
        const int pos = __ldg(offs + slab * (m + 1) + j) + atomicAdd(cursor + slab * m + j, 1);
        list[slab * per + pos] = i;
    }
}

// One warp per (key block j, slab): the list of j, ascending (the entries are
// distinct query blocks, so an entry's rank is the count of smaller ones).
__global__ void inv_sort_kernel(const int *__restrict__ offs, const int *__restrict__ in, int *__restrict__ out,
                                int m, int n, int64_t warps_total) {
    const int64_t wid = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    if (wid >= warps_total) return;
    const int64_t slab = wid / m;
    const int j = (int)(wid - slab * m);
    const int *o = offs + slab * (m + 1);
    const int64_t base = slab * (int64_t)m * n;
    const int b = o[j], L = o[j + 1] - b;
    for (int e = lane; e < L; e += 32) {
        const int x = in[base + b + e];
        int rank = 0;
        for (int f = 0; f < L; ++f) rank += in[base + b + f] < x;
        out[base + b + rank] = x;
    }
}

int grid_for(int64_t work, int threads) {
    const int64_t g = (work + threads - 1) / threads;
    return (int)(g < 148 * 16 ? (g > 0 ? g : 1) : 148 * 16);
}

}  // namespace

cudaError_t launch_bwd_prep(const Problem &p, const BwdBuffers &b, cudaStream_t stream) {
    const dim3 grid((unsigned)b.m_pad, (unsigned)p.slabs);
    bwd_prep_kernel<<<grid, 256, 0, stream>>>(
        static_cast<const __nv_bfloat16 *>(b.dout), static_cast<const __nv_bfloat16 *>(b.o_fg),
        static_cast<const __nv_bfloat16 *>(b.o_l), b.gates, b.o_cg, b.lse_cg, b.qbar, b.kbar, b.vbar, b.dgates,
        b.dfine, static_cast<__nv_bfloat16 *>(b.docg16), b.dcg, b.lse_cg_pad, static_cast<__nv_bfloat16 *>(b.q16),
        static_cast<__nv_bfloat16 *>(b.k16), static_cast<__nv_bfloat16 *>(b.v16), p.n_tokens, (int)p.m, (int)b.m_pad,
        (int)p.block_size);
    return cudaGetLastError();
}

cudaError_t launch_inverse_index(const Problem &p, const int32_t *idx, int *count, int *offs, int *cursor,
                                 int *list_tmp, int *list, uint32_t *status, cudaStream_t stream) {
    const int64_t total = p.slabs * p.m * p.top_n;
    cudaError_t e = cudaMemsetAsync(count, 0, sizeof(int) * p.slabs * p.m, stream);
    if (e == cudaSuccess) e = cudaMemsetAsync(cursor, 0, sizeof(int) * p.slabs * p.m, stream);
    if (e != cudaSuccess) return e;
    inv_count_kernel<<<grid_for(total, 256), 256, 0, stream>>>(idx, total, (int)p.m, (int)p.top_n, count, status);
    inv_scan_kernel<<<(unsigned)p.slabs, 1024, 0, stream>>>(count, offs, (int)p.m);
    inv_fill_kernel<<<grid_for(total, 256), 256, 0, stream>>>(idx, total, (int)p.m, (int)p.top_n, offs, cursor,
                                                              list_tmp);
    const int64_t warps = p.slabs * p.m;
    inv_sort_kernel<<<(unsigned)((warps * 32 + 255) / 256), 256, 0, stream>>>(offs, list_tmp, list, (int)p.m,
                                                                             (int)p.top_n, warps);
    return cudaGetLastError();
}

}  // namespace bsa

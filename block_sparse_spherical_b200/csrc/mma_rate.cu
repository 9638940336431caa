// Test hook: the issue and execution rate of tcgen05.mma (kind::f16, bf16 operands, K = 16) for
// an M x N tile, issued back to back by one thread in each of `warps` warps of one CTA. The
// fine-attention kernel's tiles are M = 64 (a query block); this measures what that shape can
// reach on the tensor pipe against M = 128, and what one issuing thread can sustain.
// Operands are zero tiles in shared memory (128-byte swizzle, K-major); each warp accumulates
// into its own tensor-memory columns (overlapping when the warps' N do not fit: a race on values
// only, never outside the allocation). The wait for completion is bounded.
#include <cstdint>

#include "bsa_internal.cuh"
#include "tc_common.cuh"

namespace bsa {
namespace {

using namespace tc;

constexpr int kRounds = 64;                // rounds of 4 MMAs (K = 64) per warp
constexpr int kSmemA = 128 * 128;          // up to 128 rows x 128 B
constexpr int kSmemB = 256 * 128;          // up to 256 rows x 128 B

__global__ void __launch_bounds__(128, 1) mma_rate_kernel(long long *cycles, int m, int n, int warps) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint8_t *A = base, *B = base + kSmemA;
    __shared__ uint64_t bar[4];
    __shared__ uint32_t tmem_base;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    for (int i = tid; i < (kSmemA + kSmemB) / 4; i += blockDim.x) reinterpret_cast<uint32_t *>(base)[i] = 0u;
    if (tid == 0) {
        for (int i = 0; i < 4; ++i) mbar_init(&bar[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 512;" ::"r"(smem_u32(&tmem_base))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_proxy_async();
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = tmem_base;
    const uint32_t idesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
    uint32_t col = (uint32_t)(warp * (512 / warps));
    if (col + (uint32_t)n > 512u) col = 512u - (uint32_t)n;
    if (warp < warps && lane == 0) {
        const uint64_t da = desc_kmajor_sw128(A), db = desc_kmajor_sw128(B);
        const long long t0 = clock64();
#pragma unroll 1
        for (int i = 0; i < kRounds; ++i)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma_bf16(tmem + col, da + 2 * kk, db + 2 * kk, idesc, 1u);
        commit(&bar[warp]);
        const long long t1 = clock64();
        bool done = false;
        while (!(done = mbar_try_wait(&bar[warp], 0u)) && clock64() - t1 < 2000000000LL) {
        }
        cycles[warp] = done ? clock64() - t0 : -1;
    }
    fence_before();
    __syncthreads();
    if (warp == 0) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 512;" ::"r"(tmem) : "memory");
    }
}

}  // namespace

cudaError_t launch_mma_rate(int m, int n, int warps, long long *cycles, cudaStream_t stream) {
    const int smem = kSmemA + kSmemB + 1024;
    cudaError_t e = cudaFuncSetAttribute(mma_rate_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    mma_rate_kernel<<<1, 128, smem, stream>>>(cycles, m, n, warps);
    return cudaGetLastError();
}

int mma_rate_mmas_per_warp() { return 4 * kRounds; }

}  // namespace bsa

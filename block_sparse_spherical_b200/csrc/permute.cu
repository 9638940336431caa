// Token-order permutation for layouts other than HEALPix NESTED.
//
// BSA cuts the sequence into contiguous blocks; with NESTED order a block is
// one parent pixel (MOSAIC note, HEALPix section). The note's ablation "BSA
// but not HEALPix (lat-lon block)" runs the same attention with blocks taken
// from a latitude-longitude grid instead; this kernel moves tokens between
// such a layout and block-contiguous order: dst[s][t] = src[s][perm[t]] for
// every slab s, whole rows of row_bytes at a time (16-byte vectors, or 4-byte
// words for rows such as the 12-byte gate triples; several rows per warp).
// HBM-bound: every byte is read once and written once.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

// T: the unit a lane moves (uint4 when rows are a multiple of 16 bytes, else 4-byte
// words). A warp moves 32 / lpr rows at a time, lpr lanes per row (lpr = the row's
// units, up to 32), so that short rows (128-byte bf16 rows: 8 lanes) keep every
// lane busy.
template <typename T>
__global__ void __launch_bounds__(256)
permute_rows_kernel(const T *__restrict__ src, T *__restrict__ dst, const int32_t *__restrict__ perm,
                    int64_t slabs, int64_t n_tokens, int units_per_row, int lpr, uint32_t *status) {
    const int lane = threadIdx.x & 31;
    const int rpw = 32 / lpr;                       // rows per warp pass
    const int sub = lane / lpr, part = lane - sub * lpr;
    const int64_t rows = slabs * n_tokens;
    const int64_t warps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    for (int64_t row0 = ((blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5) * rpw; row0 < rows;
         row0 += warps * rpw) {
        const int64_t row = row0 + sub;
        if (sub >= rpw || row >= rows) continue;
        const int64_t slab = row / n_tokens, t = row - slab * n_tokens;
        const int32_t from = __ldg(perm + t);
        if (from < 0 || from >= n_tokens) {
            if (part == 0 && status) atomicOr(status, kStatusBadIndex);
            continue;
        }
        const T *s = src + (slab * n_tokens + from) * units_per_row;
        T *d = dst + row * units_per_row;
        for (int e = part; e < units_per_row; e += lpr) d[e] = __ldg(s + e);
    }
}

}  // namespace

cudaError_t launch_permute_rows(const void *src, void *dst, const int32_t *perm, int64_t slabs, int64_t n_tokens,
                                int64_t row_bytes, uint32_t *status, cudaStream_t stream) {
    const int64_t rows = slabs * n_tokens;
    const bool vec = row_bytes % 16 == 0;
    const int units = (int)(vec ? row_bytes / 16 : row_bytes / 4);
    const int lpr = units >= 32 ? 32 : (units > 16 ? 32 : (units > 8 ? 16 : (units > 4 ? 8 : (units > 2 ? 4 : units))));
    int64_t ctas = (rows * lpr + 255) / 256;
    if (ctas > 148 * 32) ctas = 148 * 32;
    if (ctas < 1) ctas = 1;
    if (vec)
        permute_rows_kernel<uint4><<<(unsigned)ctas, 256, 0, stream>>>(
            static_cast<const uint4 *>(src), static_cast<uint4 *>(dst), perm, slabs, n_tokens, units, lpr, status);
    else
        permute_rows_kernel<uint32_t><<<(unsigned)ctas, 256, 0, stream>>>(
            static_cast<const uint32_t *>(src), static_cast<uint32_t *>(dst), perm, slabs, n_tokens, units, lpr,
            status);
    return cudaGetLastError();
}

}  // namespace bsa

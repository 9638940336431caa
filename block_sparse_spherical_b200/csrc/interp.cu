// Lat-lon -> HEALPix cross-attention interpolation, the step before BSA in the
// MOSAIC note's pipeline ("overall framework" (1), HEALPix paragraph): each
// HEALPix target pixel i attends to its neighbouring source points j of a
// latitude-longitude grid with the relative position p_ij as the query,
//   o_i = Σ_{j ∈ N_i} softmax_j((W_q p_ij)·k_j · s) v_j,   s = 1/sqrt(d).
//
// healpix_plan_kernel: one thread per NESTED pixel: its centre (the published
//   HEALPix ring formulas; face from the high bits, in-face (x, y) from the
//   interleaved low bits), the 4 x 4 block of grid points around it (rows
//   r0..r0+3, r0 = floor((90 - lat)/dlat) - 1 clamped to [0, nlat-4]; columns
//   c0-1..c0+2 wrapping in longitude, c0 = floor(lon/dlon)) and the relative
//   positions (x_j - x_i)/dlat_rad. The integer decisions use fp64.
// kappa_kernel + interp_kernel: (W_q p_ij)·k_j = p_ij·(W_qᵀ k_j), so every
//   source key is first reduced to kappa_j = W_qᵀ k_j (3 floats, once per source
//   point, into the caller's workspace); then one half-warp per target, lane j
//   holding neighbour j: logit p_ij·kappa_j, exact softmax over the 16 lanes,
//   and each lane sums d/16 channels of the v_j rows gathered from the small
//   (L2-resident) source grid; the batch loops inside, so the plan is read
//   once. fp32 arithmetic; bf16 or fp32 features.
#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int KN = 16;      // neighbours per target (4 x 4)
constexpr double kPiD = 3.14159265358979323846;

__global__ void __launch_bounds__(256)
healpix_plan_kernel(int64_t nside, int64_t nlat, int64_t nlon, int32_t *__restrict__ nbr, float *__restrict__ rel) {
    const int64_t npix = 12 * nside * nside;
    const int64_t p = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
    if (p >= npix) return;
    const int face_row[12] = {2, 2, 2, 2, 3, 3, 3, 3, 4, 4, 4, 4};
    const int face_col[12] = {1, 3, 5, 7, 0, 2, 4, 6, 1, 3, 5, 7};
    const int64_t per_face = nside * nside;
    const int f = (int)(p / per_face);
    const int64_t ipf = p - f * per_face;
    int64_t x = 0, y = 0;
    for (int b = 0; ((int64_t)1 << (2 * b)) < per_face; ++b) {
        x |= ((ipf >> (2 * b)) & 1) << b;
        y |= ((ipf >> (2 * b + 1)) & 1) << b;
    }
    const int64_t ring = face_row[f] * nside - x - y - 1;
    int64_t nr;
    double z;
    if (ring < nside) {
        nr = ring;
        z = 1.0 - (double)(nr * nr) / (3.0 * (double)per_face);
    } else if (ring > 3 * nside) {
        nr = 4 * nside - ring;
        z = -1.0 + (double)(nr * nr) / (3.0 * (double)per_face);
    } else {
        nr = nside;
        z = 4.0 / 3.0 - 2.0 * (double)ring / (3.0 * (double)nside);
    }
    double phi = (double)(face_col[f] * nr + (x - y)) * (kPiD / 4.0) / (double)nr;
    if (phi < 0.0) phi += 2.0 * kPiD;
    if (phi >= 2.0 * kPiD) phi -= 2.0 * kPiD;
    const double dlat = 180.0 / (double)(nlat - 1), dlon = 360.0 / (double)nlon;
    const double h = dlat * kPiD / 180.0;
    const double lat = asin(z) * 180.0 / kPiD, lon = phi * 180.0 / kPiD;
    const double st = sqrt(1.0 - z * z);
    const double xi0 = st * cos(phi), xi1 = st * sin(phi), xi2 = z;
    int64_t r0 = (int64_t)floor((90.0 - lat) / dlat) - 1;
    r0 = r0 < 0 ? 0 : (r0 > nlat - 4 ? nlat - 4 : r0);
    const int64_t c0 = (int64_t)floor(lon / dlon);
    for (int a = 0; a < 4; ++a) {
        const int64_t r = r0 + a;
        const double la = (90.0 - (double)r * dlat) * kPiD / 180.0;
        const double cl = cos(la), sl = sin(la);
        for (int b = 0; b < 4; ++b) {
            const int64_t c = ((c0 - 1 + b) % nlon + nlon) % nlon;
            const int64_t e = p * KN + a * 4 + b;
            nbr[e] = (int32_t)(r * nlon + c);
            const double lo = (double)c * dlon * kPiD / 180.0;
            rel[e * 3] = (float)((cl * cos(lo) - xi0) / h);
            rel[e * 3 + 1] = (float)((cl * sin(lo) - xi1) / h);
            rel[e * 3 + 2] = (float)((sl - xi2) / h);
        }
    }
}

// N consecutive elements (N = 2, 4 or 8; at an offset that is a multiple of N) as floats, with one
// 4-, 8- or 16-byte load for bf16 (two for 8 fp32), and the same for stores.
template <int N> struct VecU32;
template <> struct VecU32<1> { using type = uint32_t; };
template <> struct VecU32<2> { using type = uint2; };
template <> struct VecU32<4> { using type = uint4; };
template <int N>
__device__ __forceinline__ void loadv(const __nv_bfloat16 *p, float *f) {
    using V = typename VecU32<N / 2>::type;
    const V w = __ldg(reinterpret_cast<const V *>(p));
    const uint32_t *u = reinterpret_cast<const uint32_t *>(&w);
#pragma unroll
    for (int e = 0; e < N / 2; ++e) {
        f[2 * e] = __uint_as_float(u[e] << 16);
        f[2 * e + 1] = __uint_as_float(u[e] & 0xffff0000u);
    }
}
template <int N>
__device__ __forceinline__ void loadv(const float *p, float *f) {
#pragma unroll
    for (int e = 0; e < N; e += 2) {
        const float2 w = __ldg(reinterpret_cast<const float2 *>(p + e));
        f[e] = w.x;
        f[e + 1] = w.y;
    }
}
template <int N>
__device__ __forceinline__ void storev(__nv_bfloat16 *p, const float *f) {
    using V = typename VecU32<N / 2>::type;
    V w;
    uint32_t *u = reinterpret_cast<uint32_t *>(&w);
#pragma unroll
    for (int e = 0; e < N / 2; ++e) {
        const __nv_bfloat162 b2 = __floats2bfloat162_rn(f[2 * e], f[2 * e + 1]);
        u[e] = *reinterpret_cast<const uint32_t *>(&b2);
    }
    *reinterpret_cast<V *>(p) = w;
}
template <int N>
__device__ __forceinline__ void storev(float *p, const float *f) {
#pragma unroll
    for (int e = 0; e < N; e += 2) *reinterpret_cast<float2 *>(p + e) = make_float2(f[e], f[e + 1]);
}

// kappa[b][j][e] = s·log2(e) · Σ_c W_q[c][e] k[b][j][c]: each source key seen from position
// space, so that the logit of (i, j) is p_ij · kappa_j (= s (W_q p_ij)·k_j). One thread per
// source point (its row read with 16-byte vector loads, W_q from shared memory): an HBM stream.
template <typename T, int C>
__global__ void __launch_bounds__(256)
kappa_kernel(int64_t rows, const float *__restrict__ wq, const T *__restrict__ ksrc, float *__restrict__ kappa,
             float scale_log2) {
    constexpr int D = 32 * C;
    __shared__ float w[D * 3];
    for (int e = threadIdx.x; e < D * 3; e += blockDim.x) w[e] = __ldg(wq + e);
    __syncthreads();
    for (int64_t r = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; r < rows; r += (int64_t)gridDim.x * blockDim.x) {
        const T *kr = ksrc + r * D;
        float a0 = 0.f, a1 = 0.f, a2 = 0.f;
#pragma unroll
        for (int c0 = 0; c0 < D; c0 += 8) {
            float kv[8];
            loadv<8>(kr + c0, kv);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float *wc = w + (c0 + e) * 3;
                a0 = fmaf(wc[0], kv[e], a0);
                a1 = fmaf(wc[1], kv[e], a1);
                a2 = fmaf(wc[2], kv[e], a2);
            }
        }
        kappa[r * 3] = a0 * scale_log2;
        kappa[r * 3 + 1] = a1 * scale_log2;
        kappa[r * 3 + 2] = a2 * scale_log2;
    }
}

// One half-warp per target pixel, all batch elements in turn (the plan is read once).
// Lane j of the half holds neighbour j: its logit p_ij·kappa_j (log2 domain), then the
// softmax over the 16 lanes; each lane then sums C4 = d/16 channels of Σ_j p_j v_j.
template <typename T, int C4>
__global__ void __launch_bounds__(256)
interp_kernel(int64_t batch, int64_t n_tgt, int64_t n_src, const int32_t *__restrict__ nbr,
              const float *__restrict__ rel, const float *__restrict__ kappa, const T *__restrict__ vsrc,
              T *__restrict__ out, uint32_t *status) {
    constexpr int D = 16 * C4;
    const int lane = threadIdx.x & 31, j = lane & 15;
    const unsigned half = (lane < 16) ? 0x0000ffffu : 0xffff0000u;
    const int64_t halves = ((int64_t)gridDim.x * blockDim.x) >> 4;
    for (int64_t i = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 4; i < n_tgt; i += halves) {
        int32_t src = __ldg(nbr + i * KN + j);
        const bool bad = src < 0 || src >= n_src;
        if (bad) src = 0;
        const float *pr = rel + (i * KN + j) * 3;
        const float p0 = __ldg(pr), p1 = __ldg(pr + 1), p2 = __ldg(pr + 2);
        if (__any_sync(half, bad) && j == 0 && status) atomicOr(status, kStatusBadIndex);
        // kappa of the next batch image is loaded while this one's rows are gathered
        const float *kp0 = kappa + src * 3;
        float k0 = __ldg(kp0), k1 = __ldg(kp0 + 1), k2 = __ldg(kp0 + 2);
        for (int64_t b = 0; b < batch; ++b) {
            float lg = fmaf(p0, k0, fmaf(p1, k1, p2 * k2));
            if (b + 1 < batch) {
                const float *kp = kappa + ((b + 1) * n_src + src) * 3;
                k0 = __ldg(kp);
                k1 = __ldg(kp + 1);
                k2 = __ldg(kp + 2);
            }
            float mx = lg;
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(half, mx, off));
            const float e = exp2f(lg - mx);
            float den = e;
#pragma unroll
            for (int off = 8; off > 0; off >>= 1) den += __shfl_xor_sync(half, den, off);
            const float pj = e / den;
            float acc[C4];
#pragma unroll
            for (int c = 0; c < C4; ++c) acc[c] = 0.f;
            const T *vb = vsrc + b * n_src * D;
#pragma unroll
            for (int jj = 0; jj < KN; ++jj) {
                const float pw = __shfl_sync(half, pj, (lane & 16) | jj);
                const int32_t sj = __shfl_sync(half, src, (lane & 16) | jj);
                float vv[C4];
                loadv<C4>(vb + (int64_t)sj * D + j * C4, vv);   // one vector load per neighbour
#pragma unroll
                for (int c = 0; c < C4; ++c) acc[c] = fmaf(pw, vv[c], acc[c]);
            }
            storev<C4>(out + (b * n_tgt + i) * D + j * C4, acc);
        }
    }
}

template <typename T>
cudaError_t launch_interp_t(int64_t batch, int64_t n_tgt, int64_t n_src, int64_t d, const int32_t *nbr,
                            const float *rel, const float *wq, const void *k, const void *v, void *out, float scale,
                            float *kappa, uint32_t *status, cudaStream_t stream) {
    const float sl2 = scale * 1.4426950408889634f;
    const T *kt = static_cast<const T *>(k), *vt = static_cast<const T *>(v);
    T *ot = static_cast<T *>(out);
    const int64_t krows = batch * n_src;
    int64_t kctas = (krows + 255) / 256;
    if (kctas > 148 * 32) kctas = 148 * 32;
    if (kctas < 1) kctas = 1;
    int64_t ctas = (n_tgt * 16 + 255) / 256;
    if (ctas > 148 * 64) ctas = 148 * 64;
    if (ctas < 1) ctas = 1;
    switch (d) {
        case 32:
            kappa_kernel<T, 1><<<(unsigned)kctas, 256, 0, stream>>>(krows, wq, kt, kappa, sl2);
            interp_kernel<T, 2><<<(unsigned)ctas, 256, 0, stream>>>(batch, n_tgt, n_src, nbr, rel, kappa, vt, ot, status);
            break;
        case 64:
            kappa_kernel<T, 2><<<(unsigned)kctas, 256, 0, stream>>>(krows, wq, kt, kappa, sl2);
            interp_kernel<T, 4><<<(unsigned)ctas, 256, 0, stream>>>(batch, n_tgt, n_src, nbr, rel, kappa, vt, ot, status);
            break;
        case 128:
            kappa_kernel<T, 4><<<(unsigned)kctas, 256, 0, stream>>>(krows, wq, kt, kappa, sl2);
            interp_kernel<T, 8><<<(unsigned)ctas, 256, 0, stream>>>(batch, n_tgt, n_src, nbr, rel, kappa, vt, ot, status);
            break;
        default: return cudaErrorNotSupported;
    }
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_healpix_plan(int64_t nside, int64_t nlat, int64_t nlon, int32_t *nbr, float *rel,
                                cudaStream_t stream) {
    const int64_t npix = 12 * nside * nside;
    healpix_plan_kernel<<<(unsigned)((npix + 255) / 256), 256, 0, stream>>>(nside, nlat, nlon, nbr, rel);
    return cudaGetLastError();
}

cudaError_t launch_interp(int64_t batch, int64_t n_tgt, int64_t n_src, int64_t d, bsa_dtype dtype,
                          const int32_t *nbr, const float *rel, const float *wq, const void *k, const void *v,
                          void *out, float scale, float *kappa, uint32_t *status, cudaStream_t stream) {
    if (dtype == BSA_BF16)
        return launch_interp_t<__nv_bfloat16>(batch, n_tgt, n_src, d, nbr, rel, wq, k, v, out, scale, kappa, status,
                                              stream);
    return launch_interp_t<float>(batch, n_tgt, n_src, d, nbr, rel, wq, k, v, out, scale, kappa, status, stream);
}

}  // namespace bsa

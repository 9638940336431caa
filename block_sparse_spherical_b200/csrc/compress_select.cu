// Compressed branch (a) and top-n block selection of branch (b), BSA section
// of the MOSAIC note, in fp32 on the CUDA cores:
//
//   z_ij = s·q̄_i·k̄_j,   o_cg_i = Σ_j softmax_j(z_ij) v̄_j,
//   sel_i = top-n blocks j by (z_ij desc, j asc).
//
// One CTA owns 64 query blocks (rows) of one slab and streams the slab's k̄/v̄
// in tiles of 64 key blocks through shared memory (cp.async, double
// buffered). Per tile it forms the 64x64 logit tile in registers, runs one
// online-softmax step, merges the tile into every row's running top-n list,
// and accumulates P·v̄. The m×m logit matrix never leaves the SM.
//
// Thread layout (256 threads): warp w, half h = lane/16, tx = lane%16,
// ty = 2w+h. Thread (ty,tx) owns rows 4ty..4ty+3; its logit columns are
// tx+16jj (jj<4) and its output columns are tx*(D/16)..+D/16. A row is thus
// owned by the 16 lanes of one half-warp, which also hold that row's sorted
// top-n list (entry e = tx + 16*slot) and update it with shuffles only.
// Both products use the packed two-lane fp32 FMA of sm_100 (__ffma2_rn):
// the logits pair partial sums over even/odd feature indices, P·v̄ pairs two
// rows of P (stored transposed in shared memory) against a duplicated v̄.
#include <math_constants.h>

#include "bsa_internal.cuh"

namespace bsa {
namespace {

constexpr int BM = 64;        // query blocks per CTA
constexpr int BN = 64;        // key blocks per tile
constexpr int LDS = 68;       // padded smem row stride (floats) for 64-wide tiles

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem, bool valid) {
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    const int bytes = valid ? 16 : 0;   // 0 => zero fill
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(s), "l"(gmem), "r"(bytes));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N));
}

// (av, ai) ranks above (bv, bi): larger logit, or equal logit and lower index.
__device__ __forceinline__ bool ranks_above(float av, int ai, float bv, int bi) {
    return av > bv || (av == bv && ai < bi);
}

// Bitonic sort, within one half-warp, of one row's 64 (logit, block) pairs of
// the first key tile (4 per lane: element e = 4*tx + r), into the order
// (logit descending, block ascending). Writes the first 16*NPL of them as the
// row's initial top list: entry p at lane p%16, slot p/16.
template <int NPL>
__device__ __forceinline__ void bitonic_fill(const float *sv, const int *si, int tx, float *lv, int *li) {
    const unsigned FULL = 0xffffffffu;
    float v[4];
    int ix[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) { v[r] = sv[r]; ix[r] = si[r]; }
#pragma unroll
    for (int k = 2; k <= 64; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= 4) {                       // partner in lane tx ^ (j/4), same register
                const int lj = j >> 2;
                const bool lower = (tx & lj) == 0;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const bool desc = ((4 * tx + r) & k) == 0;
                    const float pv = __shfl_xor_sync(FULL, v[r], lj, 16);
                    const int pi = __shfl_xor_sync(FULL, ix[r], lj, 16);
                    const bool mine_better = ranks_above(v[r], ix[r], pv, pi);
                    const bool keep = (lower == desc) ? mine_better : !mine_better;
                    if (!keep) { v[r] = pv; ix[r] = pi; }
                }
            } else {                            // partner in the same lane, register r ^ j
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    if (r & j) continue;
                    const int r2 = r | j;
                    const bool desc = ((4 * tx + r) & k) == 0;
                    const bool b = ranks_above(v[r], ix[r], v[r2], ix[r2]);
                    if (b != desc) {
                        const float tv = v[r]; v[r] = v[r2]; v[r2] = tv;
                        const int ti = ix[r]; ix[r] = ix[r2]; ix[r2] = ti;
                    }
                }
            }
        }
    }
    // rank p (element p) sits in lane p/4, register p%4
#pragma unroll
    for (int h = 0; h < NPL; ++h) {
        const int pr = 16 * h + tx, src = pr >> 2, rr = pr & 3;
        float c[4];
        int d[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
            c[r] = __shfl_sync(FULL, v[r], src, 16);
            d[r] = __shfl_sync(FULL, ix[r], src, 16);
        }
        lv[h] = rr == 0 ? c[0] : rr == 1 ? c[1] : rr == 2 ? c[2] : c[3];
        li[h] = rr == 0 ? d[0] : rr == 1 ? d[1] : rr == 2 ? d[2] : d[3];
    }
}

template <int D>
__device__ __forceinline__ void load_rows(float *dst, const float *src, int row0, int m, int tid) {
    // BM rows x D floats -> dst[r*LDS + c], rows >= m zero filled
    constexpr int CPR = D / 4;                 // 16-byte chunks per row
    constexpr int TOTAL = BM * CPR;
#pragma unroll
    for (int c = tid; c < TOTAL; c += 256) {
        const int r = c / CPR, col = (c % CPR) * 4;
        const bool ok = row0 + r < m;
        const float *g = src + (int64_t)(ok ? row0 + r : 0) * D + col;
        cp_async16(dst + r * LDS + col, g, ok);
    }
}

template <int D, int NPL>
__global__ void __launch_bounds__(256, 2)
compress_select_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar,
                       const float *__restrict__ vbar, float *__restrict__ o_cg,
                       int32_t *__restrict__ idx_out, int m, int n, float scale_log2,
                       float *__restrict__ lse_out) {
    static_assert(D == 32 || D == 64, "head_dim 32 or 64");
    constexpr int DPT = D / 16;                // output columns per thread
    extern __shared__ __align__(16) float smem[];
    float *Qs = smem;                          // [BM][LDS]
    float *Ks = Qs + BM * LDS;                 // [2][BN][LDS]
    float *Vs = Ks + 2 * BN * LDS;             // [2][BN][LDS]
    float *Ps = Vs + 2 * BN * LDS;             // [BM][LDS]

    const int tid = threadIdx.x, lane = tid & 31, half = lane >> 4, tx = lane & 15;
    const int ty = 2 * (tid >> 5) + half;
    const int row0 = blockIdx.x * BM;
    const int64_t slab = blockIdx.y;
    const float *q = qbar + slab * (int64_t)m * D;
    const float *k = kbar + slab * (int64_t)m * D;
    const float *v = vbar + slab * (int64_t)m * D;

    load_rows<D>(Qs, q, row0, m, tid);
    load_rows<D>(Ks, k, 0, m, tid);
    load_rows<D>(Vs, v, 0, m, tid);
    cp_async_commit();

    float2 op[2][DPT];   // (row 4ty+2k, row 4ty+2k+1) for output column c
    float mrun[4], lrun[4];
    float lv[4][NPL];
    int li[4][NPL];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        mrun[i] = -CUDART_INF_F;
        lrun[i] = 0.f;
        if (i < 2)
#pragma unroll
            for (int c = 0; c < DPT; ++c) op[i][c] = make_float2(0.f, 0.f);
#pragma unroll
        for (int h = 0; h < NPL; ++h) { lv[i][h] = -CUDART_INF_F; li[i][h] = 0x7fffffff; }
    }
    // the list's n-th entry (the admission threshold) lives at lane tn, slot hn
    const int tn = (n - 1) & 15, hn = (n - 1) >> 4;
    const unsigned FULL = 0xffffffffu;
    const int ntiles = (m + BN - 1) / BN;

    for (int t = 0; t < ntiles; ++t) {
        const int buf = t & 1;
        if (t + 1 < ntiles) {
            load_rows<D>(Ks + (buf ^ 1) * BN * LDS, k, (t + 1) * BN, m, tid);
            load_rows<D>(Vs + (buf ^ 1) * BN * LDS, v, (t + 1) * BN, m, tid);
        }
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const float *Kt = Ks + buf * BN * LDS;
        const float *Vt = Vs + buf * BN * LDS;
        const int col0 = t * BN;

        // ---- logits of the tile: s[i][jj] for row 4ty+i, key col0+tx+16jj
        float s[4][4];
        {
            float2 sp[4][4];   // (even-feature, odd-feature) partial sums
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) sp[i][jj] = make_float2(0.f, 0.f);
#pragma unroll 1
            for (int c = 0; c < D; c += 4) {
                float4 qa[4], kb[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) qa[i] = *reinterpret_cast<const float4 *>(Qs + (4 * ty + i) * LDS + c);
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) kb[jj] = *reinterpret_cast<const float4 *>(Kt + (tx + 16 * jj) * LDS + c);
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int jj = 0; jj < 4; ++jj) {
                        sp[i][jj] = __ffma2_rn(make_float2(qa[i].x, qa[i].y), make_float2(kb[jj].x, kb[jj].y), sp[i][jj]);
                        sp[i][jj] = __ffma2_rn(make_float2(qa[i].z, qa[i].w), make_float2(kb[jj].z, kb[jj].w), sp[i][jj]);
                    }
            }
            // log2-domain logits; columns past m do not exist
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const bool ok = col0 + tx + 16 * jj < m;
#pragma unroll
                for (int i = 0; i < 4; ++i) s[i][jj] = ok ? (sp[i][jj].x + sp[i][jj].y) * scale_log2 : -CUDART_INF_F;
            }
        }

        // ---- top-n merge (rows of this half-warp)
        if (t == 0) {
            // first tile: every logit is a candidate; sort the row's 64 at once
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int sj[4];
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) sj[jj] = col0 + tx + 16 * jj;
                bitonic_fill<NPL>(s[i], sj, tx, lv[i], li[i]);
            }
        } else
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float tv = -CUDART_INF_F;
            int ti = 0x7fffffff;
#pragma unroll
            for (int h = 0; h < NPL; ++h)
                if (h == hn) { tv = lv[i][h]; ti = li[i][h]; }
            tv = __shfl_sync(FULL, tv, tn, 16);
            ti = __shfl_sync(FULL, ti, tn, 16);
            // cheap pre-filter (logit >= threshold); the exact (logit, index) order is
            // applied when the candidate is placed, so ties are still resolved exactly
            unsigned cand = 0;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj)
                if (s[i][jj] >= tv) cand |= 1u << jj;
            if (col0 + BN > m) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj)
                    if (col0 + tx + 16 * jj >= m) cand &= ~(1u << jj);
            }
            while (__any_sync(FULL, cand != 0)) {
                const unsigned ball = __ballot_sync(FULL, cand != 0);
                const unsigned mine = (ball >> (16 * half)) & 0xffffu;
                const int leader = mine ? (__ffs(mine) - 1) : 0;
                const int jj = cand ? (__ffs(cand) - 1) : 0;
                float my_s = s[i][0];
#pragma unroll
                for (int u = 1; u < 4; ++u)
                    if (jj == u) my_s = s[i][u];
                float cs = __shfl_sync(FULL, my_s, leader, 16);
                const int cj = __shfl_sync(FULL, col0 + tx + 16 * jj, leader, 16);
                if (!mine) cs = -CUDART_INF_F;         // this half has nothing to insert
                if (mine && tx == leader) cand &= cand - 1;
                // position of the candidate = number of entries ranking above it
                int pos = 0;
#pragma unroll
                for (int h = 0; h < NPL; ++h) {
                    const unsigned ab = __ballot_sync(FULL, ranks_above(lv[i][h], li[i][h], cs, cj));
                    pos += __popc((ab >> (16 * half)) & 0xffffu);
                }
                const bool insert = mine && pos < n;
                // shift entries >= pos down by one (slots high to low read old values)
#pragma unroll
                for (int h = NPL - 1; h >= 0; --h) {
                    float upv = __shfl_up_sync(FULL, lv[i][h], 1, 16);
                    int upi = __shfl_up_sync(FULL, li[i][h], 1, 16);
                    if (h > 0) {
                        const float pv = __shfl_sync(FULL, lv[i][h - 1], 15, 16);
                        const int pi = __shfl_sync(FULL, li[i][h - 1], 15, 16);
                        if (tx == 0) { upv = pv; upi = pi; }
                    }
                    const int e = tx + 16 * h;
                    if (insert && e >= pos) {
                        if (e == pos) { lv[i][h] = cs; li[i][h] = cj; }
                        else { lv[i][h] = upv; li[i][h] = upi; }
                    }
                }
                // refresh the threshold and drop candidates that no longer qualify
                float nv = -CUDART_INF_F;
                int ni = 0x7fffffff;
#pragma unroll
                for (int h = 0; h < NPL; ++h)
                    if (h == hn) { nv = lv[i][h]; ni = li[i][h]; }
                nv = __shfl_sync(FULL, nv, tn, 16);
                ni = __shfl_sync(FULL, ni, tn, 16);
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    if ((cand >> u & 1u) && !ranks_above(s[i][u], col0 + tx + 16 * u, nv, ni)) cand &= ~(1u << u);
            }
        }

        // ---- online softmax step
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            float mx = fmaxf(fmaxf(s[i][0], s[i][1]), fmaxf(s[i][2], s[i][3]));
#pragma unroll
            for (int off = 1; off < 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, off));
            const float mnew = fmaxf(mrun[i], mx);
            const float alpha = exp2f(mrun[i] - mnew);   // 0 on the first tile
            mrun[i] = mnew;
            float ls = 0.f;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const float pexp = exp2f(s[i][jj] - mnew);
                ls += pexp;
                s[i][jj] = pexp;
            }
            lrun[i] = lrun[i] * alpha + ls;
#pragma unroll
            for (int c = 0; c < DPT; ++c) {
                if (i & 1) op[i >> 1][c].y *= alpha;
                else op[i >> 1][c].x *= alpha;
            }
        }
        // P transposed: Ps[key][row], the thread's 4 rows as one 16-byte store per key
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
            *reinterpret_cast<float4 *>(Ps + (tx + 16 * jj) * LDS + 4 * ty) = make_float4(s[0][jj], s[1][jj], s[2][jj], s[3][jj]);
        __syncthreads();

        // ---- o += P · v̄_tile (rows paired: (o[0], o[1]) and (o[2], o[3]) per column)
#pragma unroll 4
        for (int j = 0; j < BN; ++j) {
            const float4 pr = *reinterpret_cast<const float4 *>(Ps + j * LDS + 4 * ty);
            float vv[DPT];
            if constexpr (DPT == 4) {
                const float4 t4 = *reinterpret_cast<const float4 *>(Vt + j * LDS + tx * 4);
                vv[0] = t4.x; vv[1] = t4.y; vv[2] = t4.z; vv[3] = t4.w;
            } else {
                const float2 t2 = *reinterpret_cast<const float2 *>(Vt + j * LDS + tx * 2);
                vv[0] = t2.x; vv[1] = t2.y;
            }
            const float2 p01 = make_float2(pr.x, pr.y), p23 = make_float2(pr.z, pr.w);
#pragma unroll
            for (int c = 0; c < DPT; ++c) {
                const float2 v2 = make_float2(vv[c], vv[c]);
                op[0][c] = __ffma2_rn(p01, v2, op[0][c]);
                op[1][c] = __ffma2_rn(p23, v2, op[1][c]);
            }
        }
        __syncthreads();   // Ps and this K/V buffer are rewritten next
    }

    // ---- finish: normalise, write o_cg and the index lists
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float l = lrun[i];
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) l += __shfl_xor_sync(FULL, l, off);
        const int r = row0 + 4 * ty + i;
        if (r < m) {
            const float inv = 1.0f / l;
            float oi[DPT];
#pragma unroll
            for (int c = 0; c < DPT; ++c) oi[c] = ((i & 1) ? op[i >> 1][c].y : op[i >> 1][c].x) * inv;
            float *dst = o_cg + (slab * m + r) * (int64_t)D + tx * DPT;
            if constexpr (DPT == 4)
                *reinterpret_cast<float4 *>(dst) = make_float4(oi[0], oi[1], oi[2], oi[3]);
            else
                *reinterpret_cast<float2 *>(dst) = make_float2(oi[0], oi[1]);
            // training: natural-log log-sum-exp of the row's scaled logits
            if (lse_out && tx == 0) lse_out[slab * m + r] = (mrun[i] + log2f(l)) * 0.69314718055994531f;
            int32_t *ix = idx_out + (slab * m + r) * (int64_t)n;
#pragma unroll
            for (int h = 0; h < NPL; ++h) {
                const int e = tx + 16 * h;
                if (e < n) ix[e] = li[i][h];
            }
        }
    }
}

template <int D, int NPL>
cudaError_t launch(const Problem &p, const float *qb, const float *kb, const float *vb, float *ocg,
                   int32_t *idx, cudaStream_t s, float *lse) {
    const size_t smem = (size_t)(BM * LDS + 4 * BN * LDS + BM * LDS) * sizeof(float);
    auto kern = compress_select_kernel<D, NPL>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((unsigned)((p.m + BM - 1) / BM), (unsigned)p.slabs);
    const float scale_log2 = p.scale * 1.4426950408889634f;
    kern<<<grid, 256, smem, s>>>(qb, kb, vb, ocg, idx, (int)p.m, (int)p.top_n, scale_log2, lse);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_compress_select(const Problem &p, const float *qbar, const float *kbar,
                                   const float *vbar, float *o_cg, int32_t *idx,
                                   cudaStream_t stream, float *lse) {
    if (p.top_n > kMaxTopN) return cudaErrorNotSupported;
    const int npl = (int)((p.top_n + 15) / 16);
    if (p.head_dim == 64) {
        switch (npl) {
            case 1: return launch<64, 1>(p, qbar, kbar, vbar, o_cg, idx, stream, lse);
            case 2: return launch<64, 2>(p, qbar, kbar, vbar, o_cg, idx, stream, lse);
            default: return launch<64, 4>(p, qbar, kbar, vbar, o_cg, idx, stream, lse);
        }
    }
    if (p.head_dim == 32) {
        switch (npl) {
            case 1: return launch<32, 1>(p, qbar, kbar, vbar, o_cg, idx, stream, lse);
            case 2: return launch<32, 2>(p, qbar, kbar, vbar, o_cg, idx, stream, lse);
            default: return launch<32, 4>(p, qbar, kbar, vbar, o_cg, idx, stream, lse);
        }
    }
    return cudaErrorNotSupported;
}

}  // namespace bsa

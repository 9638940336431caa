// Backward of softmax attention on the sm_100a tensor cores, organised by key
// tile, for the two places BSA (MOSAIC note, BSA section) runs attention
// between 64-row tiles: the selection and local branches (query block i
// against key block j, token level) and the compressed branch (query tile I
// of 64 pooled blocks against key tile J, block level, over all tiles).
//
// For one key tile J and each query tile I that attends to it (a "step"),
// with the forward's row log-sum-exp lse, the row term D = g·(dout·o) and the
// branch gate g of every query row (g = 1 for the compressed branch, whose
// incoming gradient dO_CG already carries g_CG):
//   S  = Q_I K_Jᵀ,  dP = dO_I V_Jᵀ                 (tcgen05.mma, M=N=K=64)
//   P  = exp(s·S - lse),  Pg = g·P,  dS = s·P∘(g·dP - D)      (CUDA cores)
//   dV_J += Pgᵀ dO_I,  dK_J += dSᵀ Q_I              (accumulated in TMEM)
//   dQ_I  = dS K_J                                  (TMEM, then added into an
//                                                    fp32 dq accumulator with
//                                                    vector reductions)
// Pg and dS go to shared memory as bf16 rows (the MMA's K-major 128-byte
// swizzle), which the two dV/dK MMAs read as transposed (MN-major) A operands
// and the dQ MMA as a K-major one. dK_J and dV_J are complete when the key
// tile's last step is; the epilogue writes them (token level: bf16, plus the
// key block's share dk̄/B, dv̄/B of the pooled gradients; block level: fp32).
//
// Key tiles are the units of work, handed out round-robin to two independent
// pipelines per CTA (persistent grid, one CTA per SM). Per pipeline:
//   warp p (0-1)        : MMA warp (one elected lane issues)
//   warp 2+p            : TMA copy warp: K_J and V_J per unit (two buffers),
//                         Q_I and dO_I per step (two stages)
//   warps 4+4p..7+4p    : 128 softmax threads; thread (w, lane) owns row
//                         16(w%4) + lane%16 and columns 32(lane/16)..+31 of
//                         the step's S and dP, and the same rows/columns of
//                         dQ, dK, dV
// Tensor memory (M=64 accumulators use 16 of the 32 lanes of each
// sub-partition, so two share columns in the two lane halves):
//   pipeline p: S  cols 128p..+63 lanes +0,  dP cols 128p..+63 lanes +16,
//               dK cols 128p+64..+63 lanes +0, dV cols 128p+64..+63 lanes +16
//   dQ of pipeline p: cols 256..319, lanes +16p
// Every wait on an mbarrier is bounded (2 s); on expiry the kernel records a
// timeout in the status word, the other roles stop at their next wait, the
// copies and MMAs in flight are drained, TMEM is freed and the kernel returns.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <math_constants.h>

#include "bsa_internal.cuh"
#include "tc_common.cuh"

namespace bsa {
namespace {

using namespace tc;

constexpr int BK = 64;                     // rows of a tile
constexpr int HD = 64;                     // head dim
constexpr int TILE = BK * HD * 2;          // bytes of one 64x64 bf16 tile
constexpr int NPIPE = 2;
constexpr int NTHREADS = 32 * (2 * NPIPE + 4 * NPIPE);
constexpr uint32_t TMEM_COLS = 512;

// instruction descriptors: D f32, A and B bf16, M = 64, N = 64
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(64 >> 3) << 17) |
                            ((uint32_t)(64 >> 4) << 24);
constexpr uint32_t kIdescNN = kIdesc;                          // A, B K-major
constexpr uint32_t kIdescTT = kIdesc | (1u << 15) | (1u << 16); // A, B MN-major
constexpr uint32_t kIdescNT = kIdesc | (1u << 16);              // A K-major, B MN-major

struct alignas(1024) PipeTiles {
    uint8_t k[2][TILE], v[2][TILE];        // [unit buffer]
    uint8_t q[2][TILE], o[2][TILE];        // [step stage]: Q_I and dO_I
    uint8_t pg[2][TILE], ds[2][TILE];      // [step buffer]: g·P and s·dS rows
};
struct PipeBars {
    uint64_t kv_full[2], kv_empty[2];
    uint64_t qo_full[2], qo_empty[2];
    uint64_t s_full, s_free;
    uint64_t ds_full[2], ds_empty[2];
    uint64_t dq_full, dq_free;
    uint64_t acc_full, acc_free;
    uint64_t drain;
};
struct SharedStorage {
    PipeTiles tiles[NPIPE];
    PipeBars bars[NPIPE];
    uint32_t tmem_base;
    int abort_flag;
};

struct BwdParams {
    int dense;               // 1: compressed branch (every query tile, one branch); 0: fine branches
    int64_t rows;            // rows per slab of the operand tensors (dense: m_pad, fine: N)
    int tiles;               // key tiles (= query tiles) per slab
    int64_t units;           // slabs * tiles
    int valid;               // rows per slab that exist (dense: m): later keys are masked
    int m, n, w;             // fine: blocks per slab, top-n, window (in blocks)
    int R;                   // fine: 64-row tiles per block (block_size / 64)
    const int *offs, *list;  // fine: the inverted selection (per slab: m+1 offsets, m*n entries)
    const float *lse;        // dense: [slabs*m_pad]; fine: [slabs*N][2] (FG, L)
    const float *dterm;      // D, same layout as lse
    const float *gates;      // fine: [slabs*N][3]; dense: null
    float *dq_acc;           // [slabs*rows][64], reduced into
    __nv_bfloat16 *dk, *dv;  // fine outputs [slabs*N][64]
    const float *dkbar, *dvbar;   // fine: [slabs*m_pad][64], added as 1/B shares
    int64_t m_pad;
    float inv_block;
    float *dk32, *dv32;      // dense outputs [slabs*m_pad][64]
    float scale, scale_log2;
    uint32_t *status;        // nullable
};

// Step s of the unit with slab `slab` and key tile J: its query tile and branch
// (0: selection / compressed, 1: local). Fine units run the tiles of the clamped
// window's query blocks first, then the tiles of the query blocks that selected
// J's block.
struct Unit {
    int64_t slab;
    int J, jb, lo, nloc, nsteps;   // key tile, its block, first window block, window steps
    int64_t list_base;             // fine: first list entry of block jb
};
__device__ __forceinline__ Unit unit_of(const BwdParams &p, int64_t u) {
    Unit x;
    x.slab = u / p.tiles;
    x.J = (int)(u - x.slab * p.tiles);
    if (p.dense) {
        x.nloc = 0;
        x.nsteps = p.tiles;
        x.list_base = 0;
    } else {
        x.jb = x.J / p.R;
        x.lo = max(0, x.jb - p.w);
        const int hi = min(p.m - 1, x.jb + p.w);
        x.nloc = (hi - x.lo + 1) * p.R;
        const int *o = p.offs + x.slab * (p.m + 1);
        const int b = __ldg(o + x.jb);
        x.list_base = x.slab * (int64_t)p.m * p.n + b;
        x.nsteps = x.nloc + (__ldg(o + x.jb + 1) - b) * p.R;
    }
    return x;
}
__device__ __forceinline__ int step_tile(const BwdParams &p, const Unit &x, int s, int *branch) {
    if (p.dense) {
        *branch = 0;
        return s;
    }
    if (s < x.nloc) {
        *branch = 1;
        return x.lo * p.R + s;
    }
    *branch = 0;
    const int e = s - x.nloc;
    return __ldg(p.list + x.list_base + e / p.R) * p.R + e % p.R;
}

// ------------------------------------------------------------------ roles

__device__ void loader_role(const BwdParams &p, const CUtensorMap *tq, const CUtensorMap *tk, const CUtensorMap *tv,
                            const CUtensorMap *to, PipeTiles &S, PipeBars &B, int pipe, volatile int *abort_flag) {
    const int64_t stride = NPIPE * (int64_t)gridDim.x;
    uint32_t c = 0, g = 0;
    uint64_t *last_bar[2] = {nullptr, nullptr};   // most recent K/V and Q/dO copies
    uint32_t last_par[2] = {0, 0};
    bool ok = true;
    const bool leader = elect_one();
    auto wait_w = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, wait_fast(b, par, abort_flag, p.status));
    };
    for (int64_t u = NPIPE * (int64_t)blockIdx.x + pipe; u < p.units && ok; u += stride, ++c) {
        const Unit x = unit_of(p, u);
        const int64_t base = x.slab * p.rows;
        const int kb = c & 1;
        if (!(ok = wait_w(&B.kv_empty[kb], ((c >> 1) & 1) ^ 1))) break;
        if (leader) {
            mbar_expect_tx(&B.kv_full[kb], 2 * TILE);
            tma_load_tile(S.k[kb], tk, &B.kv_full[kb], (int)(base + (int64_t)x.J * BK));
            tma_load_tile(S.v[kb], tv, &B.kv_full[kb], (int)(base + (int64_t)x.J * BK));
        }
        __syncwarp();
        last_bar[0] = &B.kv_full[kb];
        last_par[0] = (c >> 1) & 1;
        for (int s = 0; s < x.nsteps; ++s, ++g) {
            int br;
            const int I = step_tile(p, x, s, &br);
            const int st = g & 1;
            if (!(ok = wait_w(&B.qo_empty[st], ((g >> 1) & 1) ^ 1))) break;
            if (leader) {
                mbar_expect_tx(&B.qo_full[st], 2 * TILE);
                tma_load_tile(S.q[st], tq, &B.qo_full[st], (int)(base + (int64_t)I * BK));
                tma_load_tile(S.o[st], to, &B.qo_full[st], (int)(base + (int64_t)I * BK));
            }
            __syncwarp();
            last_bar[1] = &B.qo_full[st];
            last_par[1] = (g >> 1) & 1;
        }
    }
    if (!ok) {                             // let the copies in flight land before the CTA exits
        for (int i = 0; i < 2; ++i)
            if (last_bar[i]) drain_bar(last_bar[i], last_par[i]);
    }
}

__device__ void mma_role(const BwdParams &p, PipeTiles &S, PipeBars &B, uint32_t tmem, int pipe,
                         volatile int *abort_flag) {
    const int64_t stride = NPIPE * (int64_t)gridDim.x;
    const uint32_t tp = tmem + 128u * pipe;
    const uint32_t tS = tp, tdP = tp + (16u << 16), tdK = tp + 64, tdV = tp + 64 + (16u << 16);
    const uint32_t tdQ = tmem + 256 + ((16u * pipe) << 16);
    uint32_t c = 0, g = 0;
    bool ok = true;
    const bool leader = elect_one();
    auto wait_w = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, wait_fast(b, par, abort_flag, p.status));
    };
    // dV, dK and dQ of step gg (first: the unit's first step, which starts dK and dV afresh)
    auto issue_grad = [&](uint32_t gg, bool first, int kb) -> bool {
        const int b = gg & 1;
        if (!wait_w(&B.ds_full[b], (gg >> 1) & 1)) return false;
        if (first && c > 0 && !wait_w(&B.acc_free, (c - 1) & 1)) return false;
        if (gg > 0 && !wait_w(&B.dq_free, (gg - 1) & 1)) return false;
        fence_after();
        if (leader) {
            const uint64_t dpg = desc_mnmajor_sw128(S.pg[b], TILE), dds_t = desc_mnmajor_sw128(S.ds[b], TILE);
            const uint64_t dds = desc_kmajor_sw128(S.ds[b]);
            const uint64_t dO = desc_mnmajor_sw128(S.o[b], TILE), dQm = desc_mnmajor_sw128(S.q[b], TILE);
            const uint64_t dKm = desc_mnmajor_sw128(S.k[kb], TILE);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)        // K chunk kk: query rows 16kk..16kk+15
                mma_bf16(tdV, dpg + 128 * kk, dO + 128 * kk, kIdescTT, (first && kk == 0) ? 0u : 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tdK, dds_t + 128 * kk, dQm + 128 * kk, kIdescTT, (first && kk == 0) ? 0u : 1u);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)        // K chunk kk: key columns 16kk..16kk+15
                mma_bf16(tdQ, dds + 2 * kk, dKm + 128 * kk, kIdescNT, kk > 0);
            commit(&B.dq_full);
            commit(&B.ds_empty[b]);
            commit(&B.qo_empty[b]);
        }
        __syncwarp();
        return true;
    };
    for (int64_t u = NPIPE * (int64_t)blockIdx.x + pipe; u < p.units && ok; u += stride, ++c) {
        const Unit x = unit_of(p, u);
        const int kb = c & 1;
        if (!(ok = wait_w(&B.kv_full[kb], (c >> 1) & 1))) break;
        for (int s = 0; s < x.nsteps; ++s, ++g) {
            const int st = g & 1;
            if (!(ok = wait_w(&B.qo_full[st], (g >> 1) & 1))) break;
            if (g > 0 && !(ok = wait_w(&B.s_free, (g - 1) & 1))) break;
            fence_after();
            if (leader) {
                const uint64_t dq = desc_kmajor_sw128(S.q[st]), dk = desc_kmajor_sw128(S.k[kb]);
                const uint64_t dO = desc_kmajor_sw128(S.o[st]), dv = desc_kmajor_sw128(S.v[kb]);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_bf16(tS, dq + 2 * kk, dk + 2 * kk, kIdescNN, kk > 0);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) mma_bf16(tdP, dO + 2 * kk, dv + 2 * kk, kIdescNN, kk > 0);
                commit(&B.s_full);
            }
            __syncwarp();
            if (s > 0 && !(ok = issue_grad(g - 1, s == 1, kb))) break;
        }
        if (!ok) break;
        if (x.nsteps > 0 && !(ok = issue_grad(g - 1, x.nsteps == 1, kb))) break;
        if (leader) {
            commit(&B.acc_full);
            commit(&B.kv_empty[kb]);
        }
        __syncwarp();
    }
    // every MMA this warp issued must be complete before TMEM is freed
    if (leader) commit(&B.drain);
    __syncwarp();
    drain_bar(&B.drain, 0);
}

__device__ __forceinline__ void red_add_v4(float *dst, float a, float b, float c, float d) {
    asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(dst), "f"(a), "f"(b), "f"(c), "f"(d)
                 : "memory");
}

__device__ void softmax_role(const BwdParams &p, PipeTiles &S, PipeBars &B, uint32_t tmem, int pipe, int wq,
                             int lane, volatile int *abort_flag) {
    const unsigned FULL = 0xffffffffu;
    const int64_t stride = NPIPE * (int64_t)gridDim.x;
    const int ch = lane >> 4;              // column half
    const int r = 16 * wq + (lane & 15);   // row within the tile
    const uint32_t wl = (uint32_t)(32 * wq);
    const uint32_t tp = tmem + 128u * pipe;
    const uint32_t tS = tp + (wl << 16), tdP = tp + ((wl + 16) << 16);
    const uint32_t tdK = tp + 64 + (wl << 16), tdV = tp + 64 + ((wl + 16) << 16);
    const uint32_t tdQ = tmem + 256 + ((wl + 16u * pipe) << 16);
    const int prow_off = (r >> 3) * 1024 + (r & 7) * 128;
    const int sw = r & 7;
    const float sl2 = p.scale_log2, sc = p.scale;
    uint32_t c = 0, g = 0;
    bool ok = true;
    auto wait_all = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(FULL, wait_fast(b, par, abort_flag, p.status));
    };
    // dQ of step gg (query tile I of slab `slab`) into the fp32 accumulator
    auto finish_dq = [&](uint32_t gg, int64_t slab, int I) -> bool {
        if (!wait_all(&B.dq_full, gg & 1)) return false;
        fence_after();
        float a[32];
        tmem_ld16x2(tdQ, a);
        tmem_ld16x2(tdQ + 16, a + 16);
        tmem_wait_ld();
        fence_before();
        mbar_arrive(&B.dq_free);
        float *dst = p.dq_acc + (slab * p.rows + (int64_t)I * BK + r) * HD + 32 * ch;
#pragma unroll
        for (int e = 0; e < 8; ++e) red_add_v4(dst + 4 * e, a[4 * e], a[4 * e + 1], a[4 * e + 2], a[4 * e + 3]);
        return true;
    };
    for (int64_t u = NPIPE * (int64_t)blockIdx.x + pipe; u < p.units && ok; u += stride, ++c) {
        const Unit x = unit_of(p, u);
        int I_prev = 0;
        for (int s = 0; s < x.nsteps; ++s, ++g) {
            int br;
            const int I = step_tile(p, x, s, &br);
            const int64_t row = x.slab * p.rows + (int64_t)I * BK + r;
            float lse2, D, gate;
            if (p.dense) {
                lse2 = __ldg(p.lse + row) * 1.4426950408889634f;
                D = __ldg(p.dterm + row);
                gate = 1.f;
            } else {
                lse2 = __ldg(p.lse + row * 2 + br) * 1.4426950408889634f;
                D = __ldg(p.dterm + row * 2 + br);
                gate = __ldg(p.gates + row * 3 + 1 + br);
            }
            // ---- S and dP of this step
            if (!(ok = wait_all(&B.s_full, g & 1))) break;
            fence_after();
            float sv[32], dp[32];
            tmem_ld16x2(tS, sv);
            tmem_ld16x2(tS + 16, sv + 16);
            tmem_ld16x2(tdP, dp);
            tmem_ld16x2(tdP + 16, dp + 16);
            tmem_wait_ld();
            fence_before();
            mbar_arrive(&B.s_free);
            // keys past the slab's valid rows (block-level padding) take no part
            const int kvalid = p.dense ? min(32, max(0, p.valid - (x.J * BK + 32 * ch))) : 32;
            uint32_t ppk[16], dpk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                float p0 = ex2(fmaf(sv[2 * e], sl2, -lse2)), p1 = ex2(fmaf(sv[2 * e + 1], sl2, -lse2));
                if (2 * e >= kvalid) p0 = 0.f;
                if (2 * e + 1 >= kvalid) p1 = 0.f;
                const float d0 = sc * p0 * fmaf(gate, dp[2 * e], -D);
                const float d1 = sc * p1 * fmaf(gate, dp[2 * e + 1], -D);
                ppk[e] = pack_bf16x2(gate * p0, gate * p1);
                dpk[e] = pack_bf16x2(d0, d1);
            }
            // ---- g·P and s·dS rows into buffer g%2 once the MMAs of step g-2 released it
            const int b = g & 1;
            if (!(ok = wait_all(&B.ds_empty[b], ((g >> 1) & 1) ^ 1))) break;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const int chunk = 4 * ch + c4;
                const int off = prow_off + ((chunk ^ sw) << 4);
                *reinterpret_cast<uint4 *>(S.pg[b] + off) =
                    make_uint4(ppk[4 * c4], ppk[4 * c4 + 1], ppk[4 * c4 + 2], ppk[4 * c4 + 3]);
                *reinterpret_cast<uint4 *>(S.ds[b] + off) =
                    make_uint4(dpk[4 * c4], dpk[4 * c4 + 1], dpk[4 * c4 + 2], dpk[4 * c4 + 3]);
            }
            fence_proxy_async();
            fence_before();
            mbar_arrive(&B.ds_full[b]);
            // ---- dQ of the previous step
            if (s > 0 && !(ok = finish_dq(g - 1, x.slab, I_prev))) break;
            I_prev = I;
        }
        if (!ok) break;
        if (x.nsteps > 0 && !(ok = finish_dq(g - 1, x.slab, I_prev))) break;
        // ---- epilogue: dK and dV of key tile J
        if (!(ok = wait_all(&B.acc_full, c & 1))) break;
        fence_after();
        float dk[32], dv[32];
        tmem_ld16x2(tdK, dk);
        tmem_ld16x2(tdK + 16, dk + 16);
        tmem_ld16x2(tdV, dv);
        tmem_ld16x2(tdV + 16, dv + 16);
        tmem_wait_ld();
        fence_before();
        mbar_arrive(&B.acc_free);
        const int64_t krow = x.slab * p.rows + (int64_t)x.J * BK + r;
        if (p.dense) {
            float4 *k4 = reinterpret_cast<float4 *>(p.dk32 + krow * HD + 32 * ch);
            float4 *v4 = reinterpret_cast<float4 *>(p.dv32 + krow * HD + 32 * ch);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                k4[e] = make_float4(dk[4 * e], dk[4 * e + 1], dk[4 * e + 2], dk[4 * e + 3]);
                v4[e] = make_float4(dv[4 * e], dv[4 * e + 1], dv[4 * e + 2], dv[4 * e + 3]);
            }
        } else {
            // + the key block's 1/B share of the pooled gradients dk̄_J, dv̄_J
            const float *kb = p.dkbar + (x.slab * p.m_pad + x.jb) * HD + 32 * ch;
            const float *vb = p.dvbar + (x.slab * p.m_pad + x.jb) * HD + 32 * ch;
            uint4 *k4 = reinterpret_cast<uint4 *>(p.dk + krow * HD + 32 * ch);
            uint4 *v4 = reinterpret_cast<uint4 *>(p.dv + krow * HD + 32 * ch);
            const float ib = p.inv_block;
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint32_t wk[4], wv[4];
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const int cc = 8 * e + 2 * h;
                    wk[h] = pack_bf16x2(fmaf(__ldg(kb + cc), ib, dk[cc]), fmaf(__ldg(kb + cc + 1), ib, dk[cc + 1]));
                    wv[h] = pack_bf16x2(fmaf(__ldg(vb + cc), ib, dv[cc]), fmaf(__ldg(vb + cc + 1), ib, dv[cc + 1]));
                }
                k4[e] = make_uint4(wk[0], wk[1], wk[2], wk[3]);
                v4[e] = make_uint4(wv[0], wv[1], wv[2], wv[3]);
            }
        }
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
attend_bwd_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                     const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap to,
                     const BwdParams p) {
    extern __shared__ uint8_t smem_raw[];
    SharedStorage &sh = *reinterpret_cast<SharedStorage *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = &sh.abort_flag;
    if (threadIdx.x == 0) {
        sh.abort_flag = 0;
        for (int q = 0; q < NPIPE; ++q) {
            PipeBars &B = sh.bars[q];
            for (int b = 0; b < 2; ++b) {
                mbar_init(&B.kv_full[b], 1);
                mbar_init(&B.kv_empty[b], 1);
                mbar_init(&B.qo_full[b], 1);
                mbar_init(&B.qo_empty[b], 1);
                mbar_init(&B.ds_full[b], 128);
                mbar_init(&B.ds_empty[b], 1);
            }
            mbar_init(&B.s_full, 1);
            mbar_init(&B.s_free, 128);
            mbar_init(&B.dq_full, 1);
            mbar_init(&B.dq_free, 128);
            mbar_init(&B.acc_full, 1);
            mbar_init(&B.acc_free, 128);
            mbar_init(&B.drain, 1);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sh.tmem_base)),
                     "r"(TMEM_COLS)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    fence_before();
    __syncthreads();
    fence_after();
    const uint32_t tmem = sh.tmem_base;
    if (warp < NPIPE) {
        mma_role(p, sh.tiles[warp], sh.bars[warp], tmem, warp, abort_flag);
    } else if (warp < 2 * NPIPE) {
        const int q = warp - NPIPE;
        loader_role(p, &tq, &tk, &tv, &to, sh.tiles[q], sh.bars[q], q, abort_flag);
    } else {
        const int q = (warp - 2 * NPIPE) >> 2;
        softmax_role(p, sh.tiles[q], sh.bars[q], tmem, q, warp & 3, lane, abort_flag);
    }
    __syncwarp();
    fence_before();
    __syncthreads();
    if (warp == 0) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

cudaError_t launch(const BwdParams &p, const void *q, const void *k, const void *v, const void *dout,
                   int64_t total_rows, cudaStream_t stream) {
    if (total_rows > 0x7fffffffLL) return cudaErrorNotSupported;   // TMA row coordinate is int32
    CUtensorMap tq, tk, tv, to;
    if (!make_tile_map_bf16x64(&tq, q, total_rows) || !make_tile_map_bf16x64(&tk, k, total_rows) ||
        !make_tile_map_bf16x64(&tv, v, total_rows) || !make_tile_map_bf16x64(&to, dout, total_rows))
        return cudaErrorInvalidValue;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    if (p.units == 0) return cudaSuccess;
    const int64_t want = (p.units + NPIPE - 1) / NPIPE;
    const int grid = (int)(want < sms ? want : sms);
    const size_t smem = sizeof(SharedStorage) + 1024;
    cudaError_t e = cudaFuncSetAttribute(attend_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attend_bwd_tc_kernel<<<grid, NTHREADS, smem, stream>>>(tq, tk, tv, to, p);
    return cudaGetLastError();
}

BwdParams base_params(const Problem &pb, const BwdBuffers &b) {
    BwdParams p = {};
    p.m = (int)pb.m;
    p.n = (int)pb.top_n;
    p.w = (int)pb.window;
    p.m_pad = b.m_pad;
    p.inv_block = 1.f / (float)pb.block_size;
    p.scale = pb.scale;
    p.scale_log2 = pb.scale * 1.4426950408889634f;
    p.status = b.status;
    return p;
}

}  // namespace

cudaError_t launch_attend_bwd_compressed(const Problem &pb, const BwdBuffers &b, cudaStream_t stream) {
    BwdParams p = base_params(pb, b);
    p.dense = 1;
    p.R = 1;
    p.rows = b.m_pad;
    p.tiles = (int)(b.m_pad / BK);
    p.units = pb.slabs * p.tiles;
    p.valid = (int)pb.m;
    p.lse = b.lse_cg_pad;
    p.dterm = b.dcg;
    p.dq_acc = b.dqbar;
    p.dk32 = b.dkbar;
    p.dv32 = b.dvbar;
    return launch(p, b.q16, b.k16, b.v16, b.docg16, pb.slabs * b.m_pad, stream);
}

cudaError_t launch_attend_bwd_fine(const Problem &pb, const BwdBuffers &b, cudaStream_t stream) {
    if (pb.block_size % BK != 0 || pb.head_dim != HD || pb.dtype != BSA_BF16) return cudaErrorNotSupported;
    BwdParams p = base_params(pb, b);
    p.dense = 0;
    p.R = (int)(pb.block_size / BK);
    p.rows = pb.n_tokens;
    p.tiles = (int)(pb.n_tokens / BK);
    p.units = pb.slabs * p.tiles;
    p.valid = (int)pb.n_tokens;
    p.offs = b.offs;
    p.list = b.list;
    p.lse = b.lse_fine;
    p.dterm = b.dfine;
    p.gates = b.gates;
    p.dq_acc = b.dq_acc;
    p.dk = static_cast<__nv_bfloat16 *>(b.dk);
    p.dv = static_cast<__nv_bfloat16 *>(b.dv);
    p.dkbar = b.dkbar;
    p.dvbar = b.dvbar;
    return launch(p, b.q, b.k, b.v, b.dout, pb.slabs * pb.n_tokens, stream);
}

}  // namespace bsa

// Backward of softmax attention on the sm_100a tensor cores, for the two places
// BSA (MOSAIC note, BSA section) runs attention between 64-row tiles: the
// selection and local branches (query tiles against key tiles, token level) and
// the compressed branch (tiles of 64 pooled blocks, all against all).
//
// For a query tile I and a key tile J that attends to it (a "step"), with the
// forward's row log-sum-exp lse, the row term D = g·(dout·o) and the branch
// gate g of every query row (g = 1 for the compressed branch, whose incoming
// gradient dO_CG already carries g_CG):
//   S  = Q_I K_Jᵀ,  dP = dO_I V_Jᵀ                 (tcgen05.mma, M=N=K=64)
//   P  = exp(s·S - lse),  Pg = g·P,  dS = s·P∘(g·dP - D)      (CUDA cores)
//   dV_J += Pgᵀ dO_I,  dK_J += dSᵀ Q_I,  dQ_I += dS K_J
// Pg and dS go to shared memory as bf16 rows (the MMA's K-major 128-byte
// swizzle), which the dV/dK MMAs read as transposed (MN-major) A operands and
// the dQ MMA as a K-major one.
//
// Three passes of one kernel:
//   compressed (key-major, dense): units are key tiles J, steps every query tile
//     (keys past m masked); dK_J, dV_J accumulate in TMEM and are written fp32 at
//     the unit's end; dQ of each step is reduced into an fp32 dq̄ (small: one
//     row per block) with red.global.add.v4.f32.
//   fine key-major: units are key tiles J, steps the query tiles of J's block's
//     clamped window, then of the query blocks whose top-n holds it (the
//     selection inverted per slab); dK_J, dV_J accumulate in TMEM and are written
//     bf16 with the block's 1/B share of dk̄, dv̄. No dQ here.
//   fine query-major: units are query tiles I, steps the key tiles of its
//     block's selected blocks, then of its window (the forward's order); dQ_I
//     accumulates in TMEM and is written bf16 with the block's 1/B share of dq̄.
//     Recomputing S and dP here costs two MMAs a step but keeps dq free of
//     atomic reductions over the full token range.
// No atomics on dk, dv or dq: all three are bit-for-bit deterministic.
//
// Units are handed out round-robin to NPIPE independent pipelines per CTA
// (persistent grid, one CTA per SM; three by default, two with -DBSA_BWD_PIPES=2).
// Per pipeline p:
//   warp p              : MMA warp (one elected lane issues)
//   warp NPIPE+p        : TMA copy warp: the unit's two tiles (key-major: K, V;
//                         query-major: Q, dO) and the step's two (key-major: Q,
//                         dO; query-major: K, V; two stages)
//   warps C+4p..C+3+4p  : 128 softmax threads; thread (w, lane) owns row
//                         16(w%4) + lane%16 and columns 32(lane/16)..+31 of
//                         the step's S and dP, and of the unit's accumulators
// C = the control warps rounded up to whole warpgroups (4 for two pipelines, 8
// for three, where warps 6-7 only give their registers away): setmaxnreg is
// executed alike by the four warps of a warpgroup. With three pipelines the
// control warps drop to 64 registers and the softmax warps rise to 112, and the
// unit tiles and the g·P / s·dS rows are single-buffered (64 KB of shared
// memory a pipeline); with two both are double-buffered and no split is needed.
// Tensor memory (M=64 accumulators use 16 of the 32 lanes of each
// sub-partition, so two share columns in the two lane halves):
//   pipeline p: S  cols 128p..+63 lanes +0,  dP cols 128p..+63 lanes +16,
//               dK (query-major: dQ) cols 128p+64..+63 lanes +0,
//               dV cols 128p+64..+63 lanes +16
//   per-step dQ of the compressed pass, pipeline p: cols 128·NPIPE + 64(p/2)
//               ..+63, lanes +16(p%2)
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
#ifndef BSA_BWD_PIPES
#define BSA_BWD_PIPES 3
#endif
constexpr int NPIPE = BSA_BWD_PIPES;       // independent pipelines per CTA (2 or 3)
// setmaxnreg must be executed alike by the four warps of a warpgroup, so the control warps
// (an MMA and a copy warp a pipeline) fill whole warpgroups: with three pipelines warps 6-7
// only give their registers away.
constexpr int kCtrlWarps = (2 * NPIPE + 3) / 4 * 4;
constexpr int NTHREADS = 32 * (kCtrlWarps + 4 * NPIPE);
// With three pipelines the unit tiles and the g·P / s·dS rows are single-buffered (64 KB of
// shared memory a pipeline), and a register split gives the softmax threads their registers.
constexpr int UB = NPIPE == 3 ? 1 : 2;     // unit tile buffers
constexpr int DB = NPIPE == 3 ? 1 : 2;     // g·P / s·dS buffers
constexpr int kCtrlRegs = 64, kSoftRegs = 112;
constexpr int kRegsNeeded = kCtrlWarps * 32 * kCtrlRegs + 4 * NPIPE * 32 * kSoftRegs;
static_assert(NPIPE == 2 || kRegsNeeded <= 65536, "register split");
constexpr uint32_t TMEM_COLS = 512;

// instruction descriptors: D f32, A and B bf16, M = 64, N = 64
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(64 >> 3) << 17) |
                            ((uint32_t)(64 >> 4) << 24);
constexpr uint32_t kIdescNN = kIdesc;                          // A, B K-major
constexpr uint32_t kIdescTT = kIdesc | (1u << 15) | (1u << 16); // A, B MN-major
constexpr uint32_t kIdescNT = kIdesc | (1u << 16);              // A K-major, B MN-major

struct alignas(1024) PipeTiles {
    uint8_t u0[UB][TILE], u1[UB][TILE];    // [unit buffer]: K, V (key-major) or Q, dO (query-major)
    uint8_t s0[2][TILE], s1[2][TILE];      // [step stage]: Q, dO (key-major) or K, V (query-major)
    uint8_t pg[DB][TILE], ds[DB][TILE];    // [step buffer]: g·P and s·dS rows
};
struct PipeBars {
    uint64_t ut_full[2], ut_empty[2];
    uint64_t st_full[2], st_empty[2];
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
    int qmajor;              // 1: units are query tiles and the pass forms dQ only (fine branches)
    int with_dq;             // key-major pass: also form dQ per step and reduce it into dq_acc
    int64_t rows;            // rows per slab of the operand tensors (dense: m_pad, fine: N)
    int tiles;               // 64-row tiles per slab
    int64_t units;           // slabs * tiles
    int valid;               // rows per slab that exist (dense: m): later keys are masked
    int m, n, w;             // fine: blocks per slab, top-n, window (in blocks)
    int R;                   // fine: 64-row tiles per block (block_size / 64)
    const int *offs, *list;  // key-major fine: the inverted selection (per slab: m+1 offsets, m*n entries)
    const int32_t *idx;      // query-major: the selection [slabs*m][n]
    const float *lse;        // dense: [slabs*m_pad]; fine: [slabs*N][2] (FG, L)
    const float *dterm;      // D, same layout as lse
    const float *gates;      // fine: [slabs*N][3]; dense: null
    float *dq_acc;           // key-major with_dq: [slabs*rows][64], reduced into
    __nv_bfloat16 *dk, *dv;  // key-major fine outputs [slabs*N][64]
    __nv_bfloat16 *dq;       // query-major output [slabs*N][64]
    const float *dkbar, *dvbar, *dqbar;   // fine: [slabs*m_pad][64], added as 1/B shares
    int64_t m_pad;
    float inv_block;
    float *dk32, *dv32;      // dense outputs [slabs*m_pad][64]
    float scale, scale_log2;
    uint32_t *status;        // nullable
};

// A unit: tile T of slab `slab` (the key tile of a key-major pass, the query tile of
// a query-major one) and its steps. Key-major fine units run the query tiles of
// T's block's clamped window, then those of the query blocks that selected it;
// query-major units run the key tiles of the selected blocks, then of the window.
struct Unit {
    int64_t slab;
    int T, tb, lo, nloc, nsteps;   // tile, its block, first window block, window steps (key-major)
    int64_t list_base;             // key-major fine: first list entry of block tb
    const int32_t *sel;            // query-major: the selected blocks of block tb
};
struct Step {
    int tile;                      // the other side's tile
    int branch;                    // 0: selection / compressed, 1: local
    bool valid;                    // false: a selected block outside [0, m) (no keys)
};
__device__ __forceinline__ Unit unit_of(const BwdParams &p, int64_t u) {
    Unit x;
    x.slab = u / p.tiles;
    x.T = (int)(u - x.slab * p.tiles);
    x.lo = x.nloc = 0;
    x.list_base = 0;
    x.sel = nullptr;
    if (p.dense) {
        x.tb = x.T;
        x.nsteps = p.tiles;
    } else if (p.qmajor) {
        x.tb = x.T / p.R;
        x.sel = p.idx + (x.slab * p.m + x.tb) * (int64_t)p.n;
        x.nsteps = (p.n + 2 * p.w + 1) * p.R;
    } else {
        x.tb = x.T / p.R;
        x.lo = max(0, x.tb - p.w);
        const int hi = min(p.m - 1, x.tb + p.w);
        x.nloc = (hi - x.lo + 1) * p.R;
        const int *o = p.offs + x.slab * (p.m + 1);
        const int b = __ldg(o + x.tb);
        x.list_base = x.slab * (int64_t)p.m * p.n + b;
        x.nsteps = x.nloc + (__ldg(o + x.tb + 1) - b) * p.R;
    }
    return x;
}
__device__ __forceinline__ Step step_of(const BwdParams &p, const Unit &x, int s) {
    Step st;
    st.valid = true;
    if (p.dense) {
        st.tile = s;
        st.branch = 0;
    } else if (p.qmajor) {
        const int nr = p.n * p.R;
        int j;
        if (s < nr) {
            j = __ldg(x.sel + s / p.R);
            st.branch = 0;
        } else {
            j = x.tb - p.w + (s - nr) / p.R;
            st.branch = 1;
        }
        st.valid = j >= 0 && j < p.m;
        st.tile = st.valid ? j * p.R + s % p.R : x.T;   // an invalid block loads a harmless tile
    } else if (s < x.nloc) {
        st.tile = x.lo * p.R + s;
        st.branch = 1;
    } else {
        const int e = s - x.nloc;
        st.tile = __ldg(p.list + x.list_base + e / p.R) * p.R + e % p.R;
        st.branch = 0;
    }
    return st;
}

// ------------------------------------------------------------------ roles

// Unit tiles (key-major: K_T, V_T; query-major: Q_T, dO_T) per unit, two buffers;
// step tiles (key-major: Q, dO of the step's query tile; query-major: K, V of the
// step's key tile) per step, two stages.
__device__ void loader_role(const BwdParams &p, const CUtensorMap *tq, const CUtensorMap *tk, const CUtensorMap *tv,
                            const CUtensorMap *to, PipeTiles &S, PipeBars &B, int pipe, volatile int *abort_flag) {
    const int64_t stride = NPIPE * (int64_t)gridDim.x;
    const CUtensorMap *u0 = p.qmajor ? tq : tk, *u1 = p.qmajor ? to : tv;
    const CUtensorMap *s0 = p.qmajor ? tk : tq, *s1 = p.qmajor ? tv : to;
    uint32_t c = 0, g = 0;
    uint64_t *last_bar[2] = {nullptr, nullptr};   // most recent unit and step copies
    uint32_t last_par[2] = {0, 0};
    bool ok = true;
    const bool leader = elect_one();
    auto wait_w = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, wait_fast(b, par, abort_flag, p.status));
    };
    for (int64_t u = NPIPE * (int64_t)blockIdx.x + pipe; u < p.units && ok; u += stride, ++c) {
        const Unit x = unit_of(p, u);
        const int64_t base = x.slab * p.rows;
        const int kb = c % UB;
        if (!(ok = wait_w(&B.ut_empty[kb], ((c / UB) & 1) ^ 1))) break;
        if (leader) {
            mbar_expect_tx(&B.ut_full[kb], 2 * TILE);
            tma_load_tile(S.u0[kb], u0, &B.ut_full[kb], (int)(base + (int64_t)x.T * BK));
            tma_load_tile(S.u1[kb], u1, &B.ut_full[kb], (int)(base + (int64_t)x.T * BK));
        }
        __syncwarp();
        last_bar[0] = &B.ut_full[kb];
        last_par[0] = (c / UB) & 1;
        for (int s = 0; s < x.nsteps; ++s, ++g) {
            const Step stp = step_of(p, x, s);
            const int st = g & 1;
            // a selected block outside [0, m) is an error in the caller's indices; a window
            // block past either end of the sequence is the clamping, not an error
            if (leader && !stp.valid && stp.branch == 0 && p.status) atomicOr(p.status, kStatusBadIndex);
            if (!(ok = wait_w(&B.st_empty[st], ((g >> 1) & 1) ^ 1))) break;
            if (leader) {
                mbar_expect_tx(&B.st_full[st], 2 * TILE);
                tma_load_tile(S.s0[st], s0, &B.st_full[st], (int)(base + (int64_t)stp.tile * BK));
                tma_load_tile(S.s1[st], s1, &B.st_full[st], (int)(base + (int64_t)stp.tile * BK));
            }
            __syncwarp();
            last_bar[1] = &B.st_full[st];
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
    const uint32_t tdQ = tmem + 128u * NPIPE + 64u * (pipe >> 1) + ((16u * (pipe & 1)) << 16);
    uint32_t c = 0, g = 0;
    bool ok = true;
    const bool leader = elect_one();
    auto wait_w = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, wait_fast(b, par, abort_flag, p.status));
    };
    // the gradient MMAs of step gg (first: the unit's first step, which starts its
    // accumulators afresh). Key-major: dV += Pgᵀ·dO, dK += dSᵀ·Q (+ dQ = dS·K per step);
    // query-major: dQ += dS·K, accumulated in the dK columns.
    auto issue_grad = [&](uint32_t gg, bool first, int kb) -> bool {
        const int b = gg % DB, st = gg & 1;
        if (!wait_w(&B.ds_full[b], (gg / DB) & 1)) return false;
        if (first && c > 0 && !wait_w(&B.acc_free, (c - 1) & 1)) return false;
        if (p.with_dq && gg > 0 && !wait_w(&B.dq_free, (gg - 1) & 1)) return false;
        fence_after();
        if (leader) {
            const uint64_t dds = desc_kmajor_sw128(S.ds[b]);
            if (p.qmajor) {
                const uint64_t dKm = desc_mnmajor_sw128(S.s0[st], TILE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)    // K chunk kk: key columns 16kk..16kk+15
                    mma_bf16(tdK, dds + 2 * kk, dKm + 128 * kk, kIdescNT, (first && kk == 0) ? 0u : 1u);
            } else {
                const uint64_t dpg = desc_mnmajor_sw128(S.pg[b], TILE), dds_t = desc_mnmajor_sw128(S.ds[b], TILE);
                const uint64_t dO = desc_mnmajor_sw128(S.s1[st], TILE), dQm = desc_mnmajor_sw128(S.s0[st], TILE);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)    // K chunk kk: query rows 16kk..16kk+15
                    mma_bf16(tdV, dpg + 128 * kk, dO + 128 * kk, kIdescTT, (first && kk == 0) ? 0u : 1u);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tdK, dds_t + 128 * kk, dQm + 128 * kk, kIdescTT, (first && kk == 0) ? 0u : 1u);
                if (p.with_dq) {
                    const uint64_t dKm = desc_mnmajor_sw128(S.u0[kb], TILE);
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        mma_bf16(tdQ, dds + 2 * kk, dKm + 128 * kk, kIdescNT, kk > 0);
                    commit(&B.dq_full);
                }
            }
            commit(&B.ds_empty[b]);
            commit(&B.st_empty[st]);
        }
        __syncwarp();
        return true;
    };
    for (int64_t u = NPIPE * (int64_t)blockIdx.x + pipe; u < p.units && ok; u += stride, ++c) {
        const Unit x = unit_of(p, u);
        const int kb = c % UB;
        if (!(ok = wait_w(&B.ut_full[kb], (c / UB) & 1))) break;
        for (int s = 0; s < x.nsteps; ++s, ++g) {
            const int st = g & 1;
            if (!(ok = wait_w(&B.st_full[st], (g >> 1) & 1))) break;
            if (g > 0 && !(ok = wait_w(&B.s_free, (g - 1) & 1))) break;
            fence_after();
            if (leader) {
                // S = Q·Kᵀ and dP = dO·Vᵀ (Q, dO and K, V from the unit or the step tiles)
                const uint8_t *q = p.qmajor ? S.u0[kb] : S.s0[st], *k = p.qmajor ? S.s0[st] : S.u0[kb];
                const uint8_t *o = p.qmajor ? S.u1[kb] : S.s1[st], *v = p.qmajor ? S.s1[st] : S.u1[kb];
                const uint64_t dq = desc_kmajor_sw128(q), dk = desc_kmajor_sw128(k);
                const uint64_t dO = desc_kmajor_sw128(o), dv = desc_kmajor_sw128(v);
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
            commit(&B.ut_empty[kb]);
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

// 32 consecutive values as bf16 at dst: x[e] + f * add[e] (add nullable).
__device__ __forceinline__ void store_row32_bf16(__nv_bfloat16 *dst, const float *x, const float *add, float f) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        uint32_t w[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const int cc = 8 * e + 2 * h;
            const float a0 = add ? fmaf(__ldg(add + cc), f, x[cc]) : x[cc];
            const float a1 = add ? fmaf(__ldg(add + cc + 1), f, x[cc + 1]) : x[cc + 1];
            w[h] = pack_bf16x2(a0, a1);
        }
        d4[e] = make_uint4(w[0], w[1], w[2], w[3]);
    }
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
    const uint32_t tdQ = tmem + 128u * NPIPE + 64u * (pipe >> 1) + ((wl + 16u * (pipe & 1)) << 16);
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
            const Step stp = step_of(p, x, s);
            const int I = p.qmajor ? x.T : stp.tile;   // the query tile of this step
            const int64_t row = x.slab * p.rows + (int64_t)I * BK + r;
            float lse2, D, gate;
            if (p.dense) {
                lse2 = __ldg(p.lse + row) * 1.4426950408889634f;
                D = __ldg(p.dterm + row);
                gate = 1.f;
            } else {
                lse2 = __ldg(p.lse + row * 2 + stp.branch) * 1.4426950408889634f;
                D = __ldg(p.dterm + row * 2 + stp.branch);
                gate = __ldg(p.gates + row * 3 + 1 + stp.branch);
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
            // keys that take no part: past the slab's valid rows (block-level padding), or
            // of a selected block outside [0, m)
            const int kvalid = p.dense ? min(32, max(0, p.valid - (x.T * BK + 32 * ch))) : (stp.valid ? 32 : 0);
            uint32_t ppk[16], dpk[16];
            // exponents, then all exponentials, then the products: in-order issue never waits
            // on one exp-unit result while later independent ones could be queued
            {
                const float2 sc2 = make_float2(sl2, sl2), nl2 = make_float2(-lse2, -lse2);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 x = __ffma2_rn(make_float2(sv[2 * e], sv[2 * e + 1]), sc2, nl2);
                    sv[2 * e] = x.x;
                    sv[2 * e + 1] = x.y;
                }
            }
#pragma unroll
            for (int e = 0; e < 32; ++e) sv[e] = ex2(sv[e]);
            {
                const float2 g2 = make_float2(gate, gate), nd2 = make_float2(-D, -D), s2 = make_float2(sc, sc);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    float2 p2 = make_float2(2 * e < kvalid ? sv[2 * e] : 0.f, 2 * e + 1 < kvalid ? sv[2 * e + 1] : 0.f);
                    const float2 t2 = __ffma2_rn(g2, make_float2(dp[2 * e], dp[2 * e + 1]), nd2);   // g·dP − D
                    const float2 d2 = __fmul2_rn(__fmul2_rn(s2, p2), t2);                          // s·P·(g·dP − D)
                    const float2 gp = __fmul2_rn(g2, p2);
                    ppk[e] = pack_bf16x2(gp.x, gp.y);
                    dpk[e] = pack_bf16x2(d2.x, d2.y);
                }
            }
            // ---- s·dS (and g·P) rows into buffer g%2 once the MMAs of step g-2 released it
            const int b = g % DB;
            if (!(ok = wait_all(&B.ds_empty[b], ((g / DB) & 1) ^ 1))) break;
#pragma unroll
            for (int c4 = 0; c4 < 4; ++c4) {
                const int chunk = 4 * ch + c4;
                const int off = prow_off + ((chunk ^ sw) << 4);
                if (!p.qmajor)
                    *reinterpret_cast<uint4 *>(S.pg[b] + off) =
                        make_uint4(ppk[4 * c4], ppk[4 * c4 + 1], ppk[4 * c4 + 2], ppk[4 * c4 + 3]);
                *reinterpret_cast<uint4 *>(S.ds[b] + off) =
                    make_uint4(dpk[4 * c4], dpk[4 * c4 + 1], dpk[4 * c4 + 2], dpk[4 * c4 + 3]);
            }
            fence_proxy_async();
            fence_before();
            mbar_arrive(&B.ds_full[b]);
            // ---- dQ of the previous step (key-major pass with dQ)
            if (p.with_dq && s > 0 && !(ok = finish_dq(g - 1, x.slab, I_prev))) break;
            I_prev = I;
        }
        if (!ok) break;
        if (p.with_dq && x.nsteps > 0 && !(ok = finish_dq(g - 1, x.slab, I_prev))) break;
        // ---- epilogue of the unit
        if (!(ok = wait_all(&B.acc_full, c & 1))) break;
        fence_after();
        float dk[32], dv[32];
        tmem_ld16x2(tdK, dk);
        tmem_ld16x2(tdK + 16, dk + 16);
        if (!p.qmajor) {
            tmem_ld16x2(tdV, dv);
            tmem_ld16x2(tdV + 16, dv + 16);
        }
        tmem_wait_ld();
        fence_before();
        mbar_arrive(&B.acc_free);
        const int64_t trow = x.slab * p.rows + (int64_t)x.T * BK + r;
        const float *share = nullptr;          // the block's 1/B share of a pooled gradient
        if (p.qmajor) {
            // dQ of query tile T + its block's share of dq̄
            share = p.dqbar + (x.slab * p.m_pad + x.tb) * HD + 32 * ch;
            store_row32_bf16(p.dq + trow * HD + 32 * ch, dk, share, p.inv_block);
        } else if (p.dense) {
            float4 *k4 = reinterpret_cast<float4 *>(p.dk32 + trow * HD + 32 * ch);
            float4 *v4 = reinterpret_cast<float4 *>(p.dv32 + trow * HD + 32 * ch);
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                k4[e] = make_float4(dk[4 * e], dk[4 * e + 1], dk[4 * e + 2], dk[4 * e + 3]);
                v4[e] = make_float4(dv[4 * e], dv[4 * e + 1], dv[4 * e + 2], dv[4 * e + 3]);
            }
        } else {
            // dK, dV of key tile T + its block's shares of dk̄, dv̄
            share = p.dkbar + (x.slab * p.m_pad + x.tb) * HD + 32 * ch;
            store_row32_bf16(p.dk + trow * HD + 32 * ch, dk, share, p.inv_block);
            share = p.dvbar + (x.slab * p.m_pad + x.tb) * HD + 32 * ch;
            store_row32_bf16(p.dv + trow * HD + 32 * ch, dv, share, p.inv_block);
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
                mbar_init(&B.ut_full[b], 1);
                mbar_init(&B.ut_empty[b], 1);
                mbar_init(&B.st_full[b], 1);
                mbar_init(&B.st_empty[b], 1);
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
    if (warp < kCtrlWarps) {
        if constexpr (NPIPE == 3) asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
        if (warp < NPIPE) {
            mma_role(p, sh.tiles[warp], sh.bars[warp], tmem, warp, abort_flag);
        } else if (warp < 2 * NPIPE) {
            const int q = warp - NPIPE;
            loader_role(p, &tq, &tk, &tv, &to, sh.tiles[q], sh.bars[q], q, abort_flag);
        }
    } else {
        if constexpr (NPIPE == 3) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftRegs));
        const int q = (warp - kCtrlWarps) >> 2;
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
    if (NPIPE == 3) {   // the register split must fit the registers the CTA is launched with
        cudaFuncAttributes fa;
        if ((e = cudaFuncGetAttributes(&fa, attend_bwd_tc_kernel)) != cudaSuccess) return e;
        if ((int64_t)fa.numRegs * NTHREADS < kRegsNeeded || fa.maxThreadsPerBlock < NTHREADS)
            return cudaErrorInvalidConfiguration;
    }
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
    p.with_dq = 1;
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
    p.lse = b.lse_fine;
    p.dterm = b.dfine;
    p.gates = b.gates;
    p.dkbar = b.dkbar;
    p.dvbar = b.dvbar;
    p.dqbar = b.dqbar;
    // key-major pass: dK, dV of every key tile
    p.qmajor = 0;
    p.offs = b.offs;
    p.list = b.list;
    p.dk = static_cast<__nv_bfloat16 *>(b.dk);
    p.dv = static_cast<__nv_bfloat16 *>(b.dv);
    cudaError_t e = launch(p, b.q, b.k, b.v, b.dout, pb.slabs * pb.n_tokens, stream);
    if (e != cudaSuccess) return e;
    // query-major pass: dQ of every query tile
    p.qmajor = 1;
    p.idx = b.sel_idx;
    p.dq = static_cast<__nv_bfloat16 *>(b.dq);
    return launch(p, b.q, b.k, b.v, b.dout, pb.slabs * pb.n_tokens, stream);
}

}  // namespace bsa

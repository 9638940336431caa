// Selection branch (b), local branch (c) and the gated combine of the BSA
// section (MOSAIC note) on the sm_100a tensor cores: bf16 inputs, blocks of
// 64·R tokens (R = 1, 4 or 16), head_dim 64, fp32 accumulation in tensor memory.
//
// Thanks to the NESTED order every key/value tile of 64 rows is one contiguous
// 8 KB span, so each is a single TMA box (64 rows x 128 B, 128-byte swizzle)
// copied straight into the layout tcgen05.mma reads. Per 64-row query tile the
// kernel streams the tiles of its block's n selected blocks and then of its
// 2w+1 local blocks; for each key tile it runs S = Q·Kᵀ (tcgen05.mma, M=64
// N=64 K=64) into TMEM, an online softmax on the CUDA cores (lazy rescaling),
// and O += P·V (tcgen05.mma with P, bf16, read from TMEM). When the selection
// branch ends, its output is folded with the compressed branch into acc =
// g_CG·o_CG + g_FG·o_FG, held in fp32 in TMEM (the other lane half), and the
// local branch starts a fresh O; the epilogue adds g_L·o_L and stores bf16.
//
// Organisation: a persistent grid of one CTA per SM, 768 threads, four
// independent pipelines ("slots") per CTA, each working on one query tile at a
// time in its own 128 TMEM columns. Four slots give four concurrent MMA issue
// streams (one thread issues a 64x64 tcgen05.mma about every 55 cycles, half
// of what the tensor pipe takes) and let the pipelines drift out of phase so
// that their softmax phases do not all contend for the exp unit at once.
//   warp s (0-3)       : MMA warp of slot s
//   warp 4+s           : TMA copy warp of slot s: Q, then K one step ahead of V
//   warps 8+4s..11+4s  : softmax + epilogue warpgroup of slot s; with the
//                        16x32bx2 access shape a warp reads 16 rows, threads t
//                        and t+16 sharing a row (columns 0-31 and 32-63)
// The MMA and copy roles have warps of their own (a lane spinning on one
// barrier would otherwise hold up another lane of its warp) and run
// warp-wide, with uniform control flow; one elected lane issues each MMA,
// commit and copy.
// Every wait on an mbarrier is bounded (2 s); on expiry the kernel records
// a timeout in the status word, the other roles stop at their next wait,
// in-flight copies and MMAs are drained (bounded), TMEM is freed and the
// kernel returns.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "bsa_internal.cuh"
#include "tc_common.cuh"

namespace bsa {
namespace {

using namespace tc;

constexpr int BK = 64;                      // tokens per block
constexpr int HD = 64;                      // head dim
constexpr int TILE = BK * HD * 2;           // bytes of one 64x64 bf16 tile
#ifndef BSA_TC_SLOTS
#define BSA_TC_SLOTS 4
#endif
#ifndef BSA_TC_STAGES
#define BSA_TC_STAGES 2
#endif
#ifndef BSA_TC_P_TMEM
#define BSA_TC_P_TMEM 1
#endif
#ifndef BSA_TC_POLY_PAIRS
#define BSA_TC_POLY_PAIRS 0
#endif
constexpr int NSLOT = BSA_TC_SLOTS;        // independent pipelines per CTA
constexpr int NSTAGE = BSA_TC_STAGES;      // depth of the K and V rings
constexpr bool P_TMEM = BSA_TC_P_TMEM != 0;   // P·V reads P from tensor memory (else shared memory)
// of each thread's 16 pairs of softmax numerators per step, how many take the FMA-pipe exp2
// (exp2_poly2) instead of the exp unit (ex2.approx), to share the load between the two pipes
constexpr int POLY_PAIRS = BSA_TC_POLY_PAIRS;
constexpr int NTHREADS = 32 * (2 * NSLOT + 4 * NSLOT);
// Register split (setmaxnreg): the two control warpgroups (MMA issuers, loaders)
// drop to kCtrlRegs, the softmax warpgroups rise to kSoftRegs. The sum must not
// exceed what the CTA was launched with; the host checks the compiled count.
constexpr int kCtrlRegs = 48, kSoftRegs = 96;
constexpr int kRegsNeeded = 2 * NSLOT * 32 * kCtrlRegs + 4 * NSLOT * 32 * kSoftRegs;
// setmaxnreg must be executed alike by the four warps of a warpgroup: the 2·NSLOT control warps
// have to fill whole warpgroups, or a mixed one could wait forever
static_assert((2 * NSLOT) % 4 == 0, "control warps must fill whole warpgroups");
constexpr uint32_t TMEM_COLS = 512;         // 128 columns per slot
constexpr float kRescaleLog2 = 8.0f;        // lazy rescale threshold (factor 256)
constexpr int kMaxMirrors = 7;              // output copies beyond `out` (8 ranks of one node)

// Tensor-memory map of a slot (128 columns). An M=64 accumulator occupies 16
// of the 32 lanes of each sub-partition (row r in lane 32*(r/16) + r%16 + base,
// base 0 or 16), so two of them can share columns in the two lane halves.
//   O   (P·V accumulator)                       columns  0..63,  lanes +0
//   S   (Q·Kᵀ scores)                           columns  0..63,  lanes +16   (P in TMEM)
//                                               columns 64..127, lanes +0    (P in shared memory)
//   P   (softmax numerators, bf16 pairs, the A  columns 64..95 / 96..127 (buffer 0 / 1),
//        operand of P·V; two buffers)           lanes +0, same lanes as O as the MMA requires
//   acc (fp32 g_CG·o_CG + g_FG·o_FG, written    columns 64..127, lanes +16
//        and read only by the softmax threads)
constexpr uint32_t O_COL = 0, O_LANE = 0;
constexpr uint32_t S_COL = P_TMEM ? 0 : 64, S_LANE = P_TMEM ? 16 : 0;
constexpr uint32_t P_COL = 64, P_LANE = 0;
constexpr uint32_t ACC_COL = 64, ACC_LANE = 16;
static_assert(P_TMEM || (S_COL != O_COL || S_LANE != O_LANE), "S and O overlap");

constexpr int NPBUF_SMEM = P_TMEM ? 0 : 2;
struct alignas(1024) SlotTiles {
    uint8_t q[TILE];
    uint8_t k[NSTAGE][TILE];   // [stage]
    uint8_t v[NSTAGE][TILE];   // [stage]
    uint8_t p[NPBUF_SMEM > 0 ? NPBUF_SMEM : 1][NPBUF_SMEM > 0 ? TILE : 1024];   // [buffer]: P(g) in buffer g%2
};
static_assert(sizeof(SlotTiles) == (1 + 2 * NSTAGE) * TILE + (P_TMEM ? 1024 : 2 * TILE), "tile layout");

struct SlotBars {
    uint64_t q_full, q_empty;
    uint64_t p_full[2];
    uint64_t k_full[NSTAGE], k_empty[NSTAGE];
    uint64_t v_full[NSTAGE], v_empty[NSTAGE];
    uint64_t o_done[2];        // [step % 2]: P·V of that step complete
    uint64_t s_full, s_free, drain;
};

struct SharedStorage {
    SlotTiles tiles[NSLOT];
    SlotBars bars[NSLOT];
    uint32_t tmem_base;
    int abort_flag;
};

struct TcParams {
    const int32_t *idx;     // [slabs*m][n]
    const float *gates;     // [slabs*N][3]
    const float *o_cg;      // [slabs*m][64]
    __nv_bfloat16 *out;     // [slabs*N][64]
    uint32_t *status;       // nullable
    // training outputs (all null, or all set): the normalised branch outputs and the
    // log-sum-exp (natural log) of each row's scaled logits per branch, for the backward
    __nv_bfloat16 *o_fg, *o_l;   // [slabs*N][64]
    float *lse;                  // [slabs*N][2]: (FG, L)
    // further buffers that receive every output row at the same offset as `out` (the
    // sharded forward's all-gather done by the epilogue's stores, e.g. into peers' memory)
    __nv_bfloat16 *mirror[kMaxMirrors];
    int n_mirror;
    int64_t n_tokens;
    int64_t total_blocks;   // slabs * tiles query tiles (64 rows each)
    int64_t tiles;          // 64-row tiles per slab (N / 64)
    int m, n, w;            // blocks per slab, top-n, window (in blocks)
    int R, logR;            // 64-row tiles per block (block_size / 64, a power of two) and its log2
    float scale_log2;
    int64_t withhold_v_step;   // test hook, -1 = off
};

// ---------------------------------------------------------------- PTX glue

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D (TMEM) (+)= A·B with A (K-major bf16 pairs, the lanes of D) read from tensor memory.
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 16 lanes x 16 columns twice: thread t of the warp gets TMEM lane (base + t%16),
// columns [col, col+16) for t < 16 and [col+32, col+48) for t >= 16.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *r) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16], 32;"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}
// 16 lanes x 32 columns twice: thread t < 16 reads lane (base + t) columns [col, col+32),
// thread t >= 16 lane (base + t - 16) columns [col+32, col+64): one row half per thread.
__device__ __forceinline__ void tmem_ld_row32(uint32_t taddr, float *r) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15]),
          "=r"(u[16]), "=r"(u[17]), "=r"(u[18]), "=r"(u[19]), "=r"(u[20]), "=r"(u[21]), "=r"(u[22]), "=r"(u[23]),
          "=r"(u[24]), "=r"(u[25]), "=r"(u[26]), "=r"(u[27]), "=r"(u[28]), "=r"(u[29]), "=r"(u[30]), "=r"(u[31])
        : "r"(taddr));
}
// 16 lanes x 16 columns: thread t < 16 writes lane (base + t) columns [col, col+16), thread
// t >= 16 writes lane (base + t - 16) columns [col+16, col+32): one row's 32 bf16 pairs.
__device__ __forceinline__ void tmem_st16_pairs(uint32_t taddr, const uint32_t *u) {
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 16, "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
        "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float *r) {
    const uint32_t *u = reinterpret_cast<const uint32_t *>(r);
    asm volatile(
        "tcgen05.st.sync.aligned.16x32bx2.x16.b32 [%0], 32, "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
        "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
        : "memory");
}

__device__ __forceinline__ float max32(const float *s) {
    float a[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) a[i] = fmaxf(fmax3(s[4 * i], s[4 * i + 1], s[4 * i + 2]), s[4 * i + 3]);
    return fmax3(fmax3(a[0], a[1], a[2]), fmax3(a[3], a[4], a[5]), fmaxf(a[6], a[7]));
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    uint32_t r;
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
    return r;
}

// 2^x for a pair of fp32 values on the FMA pipe: Cody-Waite split x = n + f with
// n = round(x) (the 1.5·2^23 shift rounds to nearest in the low mantissa bits) and
// f in [-1/2, 1/2], 2^f from the degree-3 minimax polynomial of relative error
// 7.5e-5 (Remez exchange; exp2_fit.py gives the coefficients), and 2^n added to
// the exponent field. x is clamped at -125, so that the exponent field stays
// positive (smaller inputs give about 2^-125 instead of 0, immaterial next to a
// softmax row sum of at least 1); the kernel's x never exceeds the lazy-rescale
// threshold (2^8), far from overflow.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    x.x = fmaxf(x.x, -125.f);
    x.y = fmaxf(x.y, -125.f);
    const float2 shift = make_float2(0x1.8p23f, 0x1.8p23f);
    const float2 t = __fadd2_rn(x, shift);                         // low bits: round(x)
    const float2 n = __fadd2_rn(t, make_float2(-0x1.8p23f, -0x1.8p23f));
    const float2 f = __ffma2_rn(n, make_float2(-1.f, -1.f), x);   // x - n, exact
    float2 p = __ffma2_rn(f, make_float2(0x1.c3f76p-5f, 0x1.c3f76p-5f), make_float2(0x1.f0de1ap-3f, 0x1.f0de1ap-3f));
    p = __ffma2_rn(p, f, make_float2(0x1.62f31ap-1f, 0x1.62f31ap-1f));
    p = __ffma2_rn(p, f, make_float2(0x1.fff692p-1f, 0x1.fff692p-1f));
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// 16 consecutive values x[e]·f as bf16 at dst (32 B, 16-byte aligned).
__device__ __forceinline__ void store_row16(__nv_bfloat16 *dst, const float *x, float f) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int c = 0; c < 2; ++c)
        d4[c] = make_uint4(pack_bf16(x[8 * c] * f, x[8 * c + 1] * f), pack_bf16(x[8 * c + 2] * f, x[8 * c + 3] * f),
                           pack_bf16(x[8 * c + 4] * f, x[8 * c + 5] * f), pack_bf16(x[8 * c + 6] * f, x[8 * c + 7] * f));
}
// 32 consecutive values x[e]·f as bf16 at dst (64 B, 16-byte aligned).
__device__ __forceinline__ void store_row32(__nv_bfloat16 *dst, const float *x, float f) {
    uint4 *d4 = reinterpret_cast<uint4 *>(dst);
#pragma unroll
    for (int c = 0; c < 4; ++c)
        d4[c] = make_uint4(pack_bf16(x[8 * c] * f, x[8 * c + 1] * f), pack_bf16(x[8 * c + 2] * f, x[8 * c + 3] * f),
                           pack_bf16(x[8 * c + 4] * f, x[8 * c + 5] * f), pack_bf16(x[8 * c + 6] * f, x[8 * c + 7] * f));
}

// Shared-memory matrix descriptor, 128-byte swizzle, sm_100 descriptor version.
__device__ __forceinline__ uint64_t smem_desc(const void *tile, uint32_t lbo_bytes, uint32_t sbo_bytes) {
    const uint32_t a = smem_u32(tile);
    uint64_t d = (uint64_t)((a >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
// K-major operand (rows of 64 bf16 = 128 B, 8-row groups 1024 B apart)
__device__ __forceinline__ uint64_t desc_kmajor(const void *tile) { return smem_desc(tile, 16, 1024); }
// MN-major operand (V as [key][d]: N = d contiguous, K = key rows 128 B apart)
__device__ __forceinline__ uint64_t desc_mnmajor(const void *tile) { return smem_desc(tile, TILE, 1024); }

// instruction descriptor: D f32, A/B bf16, M=64, N=64, A K-major, B K- or MN-major
constexpr uint32_t kIdescBase = (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(64 >> 3) << 17) |
                                ((uint32_t)(64 >> 4) << 24);
constexpr uint32_t kIdescS = kIdescBase;
constexpr uint32_t kIdescPV = kIdescBase | (1u << 16);

// ------------------------------------------------------------------ roles

// Copies of one slot, issued by the copy warp's elected lane in consumption order: the query
// block's Q tile, then K one step ahead of V (K(t+1) before V(t), since S(t+1)
// is issued before P·V(t)). Step t uses the t-th selected block (t < n), then
// the window blocks i-w .. i+w; blocks outside [0, m) are loaded as block i
// and masked by the softmax. Selected indices are fetched two steps ahead.
// LOGR: log2 of the 64-row tiles per block; MODE: 0 plain, 1 training outputs, 2 mirrored
// output stores (compile-time, so that the plain forward carries none of the others' code)
template <int LOGR>
__device__ void loader_role(const TcParams &p, const CUtensorMap *tq, const CUtensorMap *tk,
                            const CUtensorMap *tv, SlotTiles &S, SlotBars &B, int slot,
                            volatile int *abort_flag) {
    constexpr int R = 1 << LOGR, lr = LOGR;
    const int NR = p.n * R, T = (2 * p.w + 1 + p.n) * R;
    const int64_t stride = NSLOT * (int64_t)gridDim.x;
    uint32_t c = 0, gk = 0, gv = 0;
    uint64_t *last_bar[3] = {nullptr, nullptr, nullptr};   // Q, K, V: most recent copy
    uint32_t last_par[3] = {0, 0, 0};
    bool ok = true;
    const bool leader = elect_one();       // issues the copies; the whole warp runs the loop
    auto wait_w = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, wait_fast(b, par, abort_flag, p.status));
    };
    for (int64_t qi = NSLOT * (int64_t)blockIdx.x + slot; qi < p.total_blocks && ok; qi += stride, ++c) {
        // query tile within its slab (a slab holds tiles = m*R tiles, so the tile's
        // block row in idx is qi >> log2 R and its first token row is 64*qi)
        const int qt = (int)((uint32_t)qi % (uint32_t)p.tiles), i = qt >> lr;
        const int64_t base = (qi - qt) * BK;
        const int32_t *ix = p.idx + (qi >> lr) * (int64_t)p.n;
        // key tile of step t: tile t%R of the (t/R)-th selected block, then of window block
        // i-w+(t-nR)/R; blocks outside [0, m) are loaded as the query tile and masked
        auto tile_of = [&](int t, int jsel) -> int {
            const int j = t < NR ? jsel : i - p.w + ((t - NR) >> lr);
            return (j >= 0 && j < p.m) ? (j << lr) + (t & (R - 1)) : qt;
        };
        auto sel_at = [&](int u) -> int { return u < NR ? __ldg(ix + (u >> lr)) : 0; };
        int jq[3];                          // selected blocks of steps t, t+1, t+2 (ring)
        jq[0] = sel_at(0);
        jq[1] = sel_at(1);
        jq[2] = sel_at(2);
        // Q of this query block (single buffer: freed by the previous block's last S)
        if (!(ok = wait_w(&B.q_empty, (c & 1) ^ 1))) break;
        if (leader) {
            mbar_expect_tx(&B.q_full, TILE);
            tma_load_tile(S.q, tq, &B.q_full, (int)(base + (int64_t)qt * BK));
        }
        __syncwarp();
        last_bar[0] = &B.q_full;
        last_par[0] = c & 1;
        int jv = 0;                         // block of the next V copy
        auto issue_k = [&](int t, int j) -> bool {
            if (leader && t < NR && (t & (R - 1)) == 0 && (j < 0 || j >= p.m) && p.status)
                atomicOr(p.status, kStatusBadIndex);
            const int st = gk % NSTAGE;
            if (!wait_w(&B.k_empty[st], ((gk / NSTAGE) & 1) ^ 1)) return false;
            if (leader) {
                mbar_expect_tx(&B.k_full[st], TILE);
                tma_load_tile(S.k[st], tk, &B.k_full[st], (int)(base + (int64_t)tile_of(t, j) * BK));
            }
            __syncwarp();
            last_bar[1] = &B.k_full[st];
            last_par[1] = (gk / NSTAGE) & 1;
            ++gk;
            return true;
        };
        auto issue_v = [&](int t, int j) -> bool {
            const int st = gv % NSTAGE;
            if (!wait_w(&B.v_empty[st], ((gv / NSTAGE) & 1) ^ 1)) return false;
            if (!((int64_t)gv == p.withhold_v_step && blockIdx.x == 0 && slot == 0)) {   // test hook
                if (leader) {
                    mbar_expect_tx(&B.v_full[st], TILE);
                    tma_load_tile(S.v[st], tv, &B.v_full[st], (int)(base + (int64_t)tile_of(t, j) * BK));
                }
                __syncwarp();
                last_bar[2] = &B.v_full[st];
                last_par[2] = (gv / NSTAGE) & 1;
            }
            ++gv;
            return true;
        };
        if (!(ok = issue_k(0, jq[0]))) break;
        jv = jq[0];
        for (int t = 0; t < T; ++t) {
            const int jk = jq[(t + 1) % 3];   // index of step t+1
            jq[(t + 3) % 3] = t + 3 < NR ? sel_at(t + 3) : jq[t % 3];
            // (the slot just refilled held step t's index, already used by K(t) and kept in jv)
            if (t + 1 < T && !(ok = issue_k(t + 1, jk))) break;
            if (!(ok = issue_v(t, jv))) break;
            jv = jk;
        }
    }
    if (!ok) {                             // let the copies in flight land before the CTA exits
        for (int s2 = 0; s2 < 3; ++s2)
            if (last_bar[s2]) drain_bar(last_bar[s2], last_par[s2]);
    }
}

template <int LOGR>
__device__ void mma_role(const TcParams &p, SlotTiles &S, SlotBars &B, uint32_t tmem_slot, int slot,
                         volatile int *abort_flag) {
    constexpr int R = 1 << LOGR;
    const int NR = p.n * R, T = (2 * p.w + 1 + p.n) * R;
    const int64_t stride = NSLOT * (int64_t)gridDim.x;
    const uint32_t tS = tmem_slot + S_COL + (S_LANE << 16), tO = tmem_slot + O_COL + (O_LANE << 16);
    const uint32_t tP = tmem_slot + P_COL + (P_LANE << 16);   // P buffer b at + 32*b (P in TMEM)
    // shared-memory descriptors of every operand tile, computed once
    const uint64_t dq = desc_kmajor(S.q);
    const uint64_t dk0 = desc_kmajor(S.k[0]), dv0 = desc_mnmajor(S.v[0]);   // stage s: + s*TILE/16
    const uint64_t dp0 = desc_kmajor(S.p[0]), dp1 = desc_kmajor(S.p[NPBUF_SMEM > 1 ? 1 : 0]);
    uint32_t c = 0, g = 0;
    bool ok = true;
    const bool leader = elect_one();       // issues MMAs and commits; the whole warp runs the loop
    auto wait_w = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, wait_fast(b, par, abort_flag, p.status));
    };
    for (int64_t qi = NSLOT * (int64_t)blockIdx.x + slot; qi < p.total_blocks && ok; qi += stride, ++c) {
        if (!(ok = wait_w(&B.q_full, c & 1))) break;
        // S(gs) = Q·K(gs)ᵀ; needs K loaded and the previous S read out of TMEM
        auto issue_s = [&](uint32_t gs) -> bool {
            const int ks = gs % NSTAGE;
            if (!wait_w(&B.k_full[ks], (gs / NSTAGE) & 1)) return false;
            if (gs > 0 && !wait_w(&B.s_free, (gs - 1) & 1)) return false;
            fence_after();
            const uint64_t dk = dk0 + (uint64_t)(ks * (TILE >> 4));
            if (leader) {
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) tc_mma(tS, dq + 2 * kk, dk + 2 * kk, kIdescS, kk > 0);
                commit(&B.s_full);
                commit(&B.k_empty[ks]);
            }
            __syncwarp();
            return true;
        };
        if (!(ok = issue_s(g))) break;
        if (T == 1 && leader) commit(&B.q_empty);
        for (int t = 0; t < T; ++t, ++g) {
            if (t + 1 < T) {                       // the next S runs while this step's softmax does
                if (!(ok = issue_s(g + 1))) break;
                if (t + 2 == T && leader) commit(&B.q_empty);
            }
            const int vs = g % NSTAGE, pb = g & 1;
            if (!(ok = wait_w(&B.p_full[pb], (g >> 1) & 1))) break;
            if (!(ok = wait_w(&B.v_full[vs], (g / NSTAGE) & 1))) break;
            fence_after();
            const uint32_t acc0 = (t == 0 || t == NR) ? 0u : 1u;   // each branch starts a fresh O
            const uint64_t dv = dv0 + (uint64_t)(vs * (TILE >> 4));
            const uint64_t dp = pb ? dp1 : dp0;
            if (leader) {
                if (P_TMEM) {
                    // K chunk kk (16 keys) of P = 8 columns of bf16 pairs
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk)
                        tc_mma_ts(tO, tP + 32u * pb + 8u * kk, dv + 128 * kk, kIdescPV, kk ? 1u : acc0);
                } else {
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) tc_mma(tO, dp + 2 * kk, dv + 128 * kk, kIdescPV, kk ? 1u : acc0);
                }
                commit(&B.o_done[pb]);
                commit(&B.v_empty[vs]);
            }
            __syncwarp();
        }
    }
    // every MMA this thread issued must be complete before TMEM is freed
    if (leader) commit(&B.drain);
    __syncwarp();
    drain_bar(&B.drain, 0);
}

// Softmax warpgroup of a slot. Thread (wq, lane): row r = 16*wq + lane%16,
// columns 32*(lane/16) .. +31 of the query block's S and O.
template <int LOGR, int MODE>
__device__ void softmax_role(const TcParams &p, SlotTiles &S, SlotBars &B, uint32_t tmem_slot, int slot,
                             int wq, int lane, volatile int *abort_flag) {
    const unsigned FULL = 0xffffffffu;
    constexpr int R = 1 << LOGR, lr = LOGR;
    const int NR = p.n * R, T = (2 * p.w + 1 + p.n) * R;
    const int ch = lane >> 4;              // column half of the row
    const int r = 16 * wq + (lane & 15);   // row within the query block
    const uint32_t wl = (uint32_t)(32 * wq);   // this warp's sub-partition
    const uint32_t tS = tmem_slot + S_COL + ((wl + S_LANE) << 16);
    const uint32_t tO = tmem_slot + O_COL + ((wl + O_LANE) << 16);
    const uint32_t tA = tmem_slot + ACC_COL + ((wl + ACC_LANE) << 16);
    const uint32_t tP = tmem_slot + P_COL + ((wl + P_LANE) << 16);
    const int prow_off = (r >> 3) * 1024 + (r & 7) * 128;
    const int sw = r & 7;
    const float sl2 = p.scale_log2;
    const int64_t stride = NSLOT * (int64_t)gridDim.x;
    uint32_t g = 0;
    bool ok = true;
    auto wait_all = [&](uint64_t *b, uint32_t par) -> bool {
        const bool mine = wait_fast(b, par, abort_flag, p.status);
        return __all_sync(FULL, mine);
    };
    // selected blocks of query tile q (its block's index row)
    auto sel_row = [&](int64_t q) -> const int32_t * { return p.idx + (q >> lr) * (int64_t)p.n; };
    int j0 = 0, j1 = 0;                    // this lane's two selected indices of the next query tile
    {
        const int64_t q0 = NSLOT * (int64_t)blockIdx.x + slot;
        if (q0 < p.total_blocks) {
            const int32_t *ix = sel_row(q0);
            if (lane < p.n) j0 = __ldg(ix + lane);
            if (lane + 32 < p.n) j1 = __ldg(ix + lane + 32);
        }
    }
    for (int64_t qi = NSLOT * (int64_t)blockIdx.x + slot; qi < p.total_blocks && ok; qi += stride) {
        const int qt = (int)((uint32_t)qi % (uint32_t)p.tiles), i = qt >> lr;   // tile within the slab, its block
        const int64_t tok = qi * BK + r;
        const float *gp = p.gates + tok * 3;
        const float g_cg = __ldg(gp), g_fg = __ldg(gp + 1), g_l = __ldg(gp + 2);
        const float *ocg = p.o_cg + (qi >> lr) * (int64_t)HD + 32 * ch;
        asm volatile("prefetch.global.L1 [%0];" ::"l"(ocg));
        // validity of the n selected blocks of this query block, as a bit mask
        // (its indices were fetched during the previous query block)
        const unsigned lo = __ballot_sync(FULL, j0 >= 0 && j0 < p.m);
        const unsigned hi = __ballot_sync(FULL, j1 >= 0 && j1 < p.m);
        const uint64_t selmask = ((uint64_t)hi << 32) | lo;
        {
            const int64_t qn = qi + stride;
            j0 = j1 = 0;
            if (qn < p.total_blocks) {
                const int32_t *ix = sel_row(qn);
                if (lane < p.n) j0 = __ldg(ix + lane);
                if (lane + 32 < p.n) j1 = __ldg(ix + lane + 32);
            }
        }
        float m_used = -INFINITY, l_run = 0.f, l_sel = 0.f, m_sel = -INFINITY;
        for (int t = 0; t < T; ++t, ++g) {
            bool valid;
            if (t < NR) {
                valid = (selmask >> (t >> lr)) & 1u;
            } else {
                const int j = i - p.w + ((t - NR) >> lr);
                valid = j >= 0 && j < p.m;
            }
            if (t == NR) {                     // the local branch starts afresh
                l_sel = l_run;
                m_sel = m_used;
                l_run = 0.f;
                m_used = -INFINITY;
            }
            // ---- scores of this step
            if (!(ok = wait_all(&B.s_full, g & 1))) break;
            fence_after();
            float s[32];
            tmem_ld_row32(tS, s);
            tmem_wait_ld();
            fence_before();
            mbar_arrive(&B.s_free);            // every softmax thread arrives (count 128)
            // ---- softmax numerators against the (lazily updated) running max
            float mx = valid ? max32(s) : -INFINITY;
            mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16)) * sl2;
            const bool need = valid && m_used != -INFINITY && mx > m_used + kRescaleLog2;
            const float m_old = m_used;
            if (valid && (m_used == -INFINITY || need)) m_used = mx;
            uint32_t pk[16];
            float ls = 0.f;
            if (valid) {
                // p = 2^(s·scale·log2e − m), two columns per packed FMA. In three phases (all
                // exponents, then all exponentials, then packing and the sums), so that the
                // warp's in-order issue never waits on one exp-unit result while later
                // independent exponentials could still be queued
                const float2 sc2 = make_float2(sl2, sl2), nm2 = make_float2(-m_used, -m_used);
                float2 x[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) x[c] = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), sc2, nm2);
#pragma unroll
                for (int c = 0; c < 16; ++c) x[c] = (c < POLY_PAIRS) ? exp2_poly2(x[c]) : make_float2(ex2(x[c].x), ex2(x[c].y));
                float2 acc2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    pk[c] = pack_bf16(x[c].x, x[c].y);
                    acc2[c & 1] = __fadd2_rn(acc2[c & 1], x[c]);
                }
                const float2 t2 = __fadd2_rn(acc2[0], acc2[1]);
                ls = t2.x + t2.y;
            } else {
#pragma unroll
                for (int c = 0; c < 16; ++c) pk[c] = 0u;
            }
            // ---- O is touched only at the branch switch or to rescale: then P·V(g-1)
            //      must be complete
            // (S(g) complete implies P·V(g-2) complete: one thread issues both, in order,
            //  so the two-barrier parity below cannot alias)
            const bool touch_o = (t == NR) || __any_sync(FULL, need);
            if (touch_o && g > 0 && !(ok = wait_all(&B.o_done[(g - 1) & 1], ((g - 1) >> 1) & 1))) break;
            fence_after();
            if (t == NR) {
                // close the selection branch: acc = g_CG·o_CG + g_FG·o_FG, kept in fp32 in
                // this row's lanes of the other lane half until the epilogue
                const float l = l_sel + __shfl_xor_sync(FULL, l_sel, 16);
                const float inv = l > 0.f ? g_fg / l : 0.f;
                if constexpr (MODE == 1)       // training: the row log-sum-exp of o_FG
                    if (ch == 0) p.lse[tok * 2] = (m_sel + __log2f(l)) * 0.69314718055994531f;
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {   // 16 columns at a time (register pressure)
                    float a[16];
                    tmem_ld16(tO + 16 * hh, a);
                    tmem_wait_ld();
                    if constexpr (MODE == 1) {     // training: o_FG itself
                        const float inv1 = l > 0.f ? 1.f / l : 0.f;
                        store_row16(p.o_fg + tok * HD + 32 * ch + 16 * hh, a, inv1);
                    }
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {   // o_cg: one 256-byte row per query block
                        const float4 c4 = __ldg(reinterpret_cast<const float4 *>(ocg) + 4 * hh + e4);
                        a[4 * e4] = fmaf(g_cg, c4.x, a[4 * e4] * inv);
                        a[4 * e4 + 1] = fmaf(g_cg, c4.y, a[4 * e4 + 1] * inv);
                        a[4 * e4 + 2] = fmaf(g_cg, c4.z, a[4 * e4 + 2] * inv);
                        a[4 * e4 + 3] = fmaf(g_cg, c4.w, a[4 * e4 + 3] * inv);
                    }
                    tmem_st16(tA + 16 * hh, a);
                }
                tmem_wait_st();
            } else if (touch_o) {
                // rows whose running max grew by more than 2^8: rescale their O and sum
                const float alpha = need ? ex2(m_old - m_used) : 1.f;
#pragma unroll
                for (int cc = 0; cc < 2; ++cc) {
                    float o[16];
                    tmem_ld16(tO + 16 * cc, o);
                    tmem_wait_ld();
#pragma unroll
                    for (int e = 0; e < 16; ++e) o[e] *= alpha;
                    tmem_st16(tO + 16 * cc, o);
                }
                tmem_wait_st();
                l_run *= alpha;
            }
            l_run += ls;
            // ---- P (this thread's 32 columns of the row) -> buffer g%2. Its last reader,
            //      P·V(g-2), was issued before S(g) by the same thread, and a commit tracks
            //      every earlier MMA of its thread, so S(g) complete (waited above) means
            //      P·V(g-2) has released the buffer: no wait of its own
            const int pb = g & 1;
            if (P_TMEM) {
                // P (bf16 pairs) into this row's lanes of P buffer pb: the A operand of P·V
                tmem_st16_pairs(tP + 32u * pb, pk);
                tmem_wait_st();
            } else {
                uint8_t *prow = S.p[NPBUF_SMEM > 1 ? pb : 0] + prow_off;
#pragma unroll
                for (int c4 = 0; c4 < 4; ++c4) {
                    const int chunk = 4 * ch + c4;
                    const uint4 v4 = make_uint4(pk[4 * c4], pk[4 * c4 + 1], pk[4 * c4 + 2], pk[4 * c4 + 3]);
                    *reinterpret_cast<uint4 *>(prow + ((chunk ^ sw) << 4)) = v4;
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            }
            fence_before();
            mbar_arrive(&B.p_full[pb]);        // every softmax thread arrives (count 128)
        }
        if (!ok) break;
        // ---- epilogue: out = acc + g_L·o_L
        if (!(ok = wait_all(&B.o_done[(g - 1) & 1], ((g - 1) >> 1) & 1))) break;
        fence_after();
        const float l = l_run + __shfl_xor_sync(FULL, l_run, 16);
        const float inv = l > 0.f ? g_l / l : 0.f;
        if constexpr (MODE == 1) {             // training: o_L and its row log-sum-exp
            float o[32];
            tmem_ld16(tO, o);
            tmem_ld16(tO + 16, o + 16);
            tmem_wait_ld();
            store_row32(p.o_l + tok * HD + 32 * ch, o, l > 0.f ? 1.f / l : 0.f);
            if (ch == 0) p.lse[tok * 2 + 1] = (m_used + __log2f(l)) * 0.69314718055994531f;
        }
        uint4 *d4 = reinterpret_cast<uint4 *>(p.out + tok * HD + 32 * ch);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
            float o[16], a[16];
            tmem_ld16(tO + 16 * cc, o);
            tmem_ld16(tA + 16 * cc, a);
            tmem_wait_ld();
            uint32_t w8[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
                w8[e] = pack_bf16(fmaf(o[2 * e], inv, a[2 * e]), fmaf(o[2 * e + 1], inv, a[2 * e + 1]));
            const uint4 lo4 = make_uint4(w8[0], w8[1], w8[2], w8[3]), hi4 = make_uint4(w8[4], w8[5], w8[6], w8[7]);
            d4[2 * cc] = lo4;
            d4[2 * cc + 1] = hi4;
            if constexpr (MODE == 2) {
                for (int mi = 0; mi < p.n_mirror; ++mi) {
                    uint4 *m4 = reinterpret_cast<uint4 *>(p.mirror[mi] + tok * HD + 32 * ch);
                    m4[2 * cc] = lo4;
                    m4[2 * cc + 1] = hi4;
                }
            }
        }
        fence_before();
    }
}

template <int LOGR, int MODE>
__global__ void __launch_bounds__(NTHREADS, 1)
attend_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    SharedStorage &sh = *reinterpret_cast<SharedStorage *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    volatile int *abort_flag = &sh.abort_flag;

    if (threadIdx.x == 0) {
        sh.abort_flag = 0;
        for (int s = 0; s < NSLOT; ++s) {
            SlotBars &B = sh.bars[s];
            mbar_init(&B.q_full, 1);
            mbar_init(&B.q_empty, 1);
            for (int b = 0; b < 2; ++b) {
                mbar_init(&B.p_full[b], 128);
            }
            for (int b = 0; b < NSTAGE; ++b) {
                mbar_init(&B.k_full[b], 1);
                mbar_init(&B.k_empty[b], 1);
                mbar_init(&B.v_full[b], 1);
                mbar_init(&B.v_empty[b], 1);
            }
            mbar_init(&B.o_done[0], 1);
            mbar_init(&B.o_done[1], 1);
            mbar_init(&B.s_full, 1);
            mbar_init(&B.s_free, 128);
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
    static_assert(128 * NSLOT <= (int)TMEM_COLS, "TMEM columns");

    if (warp < 2 * NSLOT) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtrlRegs));
        const int slot = warp % NSLOT;
        if (warp < NSLOT)
            mma_role<LOGR>(p, sh.tiles[slot], sh.bars[slot], tmem + 128u * slot, slot, abort_flag);
        else
            loader_role<LOGR>(p, &tq, &tk, &tv, sh.tiles[slot], sh.bars[slot], slot, abort_flag);
    } else {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kSoftRegs));
        const int slot = (warp - 2 * NSLOT) >> 2;
        softmax_role<LOGR, MODE>(p, sh.tiles[slot], sh.bars[slot], tmem + 128u * slot, slot, warp & 3, lane,
                                 abort_flag);
    }
    __syncwarp();                          // reconverge role lanes before the CTA barrier

    fence_before();
    __syncthreads();
    if (warp == 0) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

// --------------------------------------------------------------- host side

bool make_tile_map(CUtensorMap *map, const void *base, uint64_t rows) {
    return make_tile_map_bf16x64(map, base, rows);
}

// Test hook: y = exp2_poly2(x) (poly != 0) or ex2.approx(x), elementwise.
__global__ void exp2_eval_kernel(const float *__restrict__ x, float *__restrict__ y, int64_t n, int poly) {
    for (int64_t i = 2 * (blockIdx.x * (int64_t)blockDim.x + threadIdx.x); i < n;
         i += 2 * (int64_t)gridDim.x * blockDim.x) {
        const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
        const float2 e = poly ? exp2_poly2(v) : make_float2(ex2(v.x), ex2(v.y));
        y[i] = e.x;
        if (i + 1 < n) y[i + 1] = e.y;
    }
}

template <int LOGR, int MODE>
cudaError_t launch_kernel(const CUtensorMap &tq, const CUtensorMap &tk, const CUtensorMap &tv, const TcParams &p,
                          int grid, cudaStream_t stream) {
    auto kern = attend_tc_kernel<LOGR, MODE>;
    const size_t smem = sizeof(SharedStorage) + 1024;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // The register split must fit the registers the CTA is launched with,
    // otherwise setmaxnreg.inc would wait forever: refuse to launch instead.
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    if ((int64_t)fa.numRegs * NTHREADS < kRegsNeeded || fa.maxThreadsPerBlock < NTHREADS)
        return cudaErrorInvalidConfiguration;
    kern<<<grid, NTHREADS, smem, stream>>>(tq, tk, tv, p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_exp2_eval(const float *x, float *y, int64_t n, int poly, cudaStream_t stream) {
    int64_t ctas = (n / 2 + 255) / 256 + 1;
    if (ctas > 148 * 16) ctas = 148 * 16;
    exp2_eval_kernel<<<(unsigned)ctas, 256, 0, stream>>>(x, y, n, poly);
    return cudaGetLastError();
}

cudaError_t launch_attend_tc(const Problem &pb, const void *q, const void *k, const void *v,
                             const float *gates, const float *o_cg, const int32_t *idx, void *out,
                             uint32_t *status, cudaStream_t stream, void *o_fg, void *o_l, float *lse,
                             void *const *mirrors, int n_mirrors) {
    if (pb.dtype != BSA_BF16 || pb.block_size % BK != 0 || pb.head_dim != HD) return cudaErrorNotSupported;
    const int64_t rows = pb.slabs * pb.n_tokens;
    if (rows > 0x7fffffffLL) return cudaErrorNotSupported;       // TMA row coordinate is int32
    CUtensorMap tq, tk, tv;
    if (!make_tile_map(&tq, q, rows) || !make_tile_map(&tk, k, rows) || !make_tile_map(&tv, v, rows))
        return cudaErrorInvalidValue;        // driver entry point missing or tensor map rejected
    TcParams p;
    p.idx = idx;
    p.gates = gates;
    p.o_cg = o_cg;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.status = status;
    p.o_fg = static_cast<__nv_bfloat16 *>(o_fg);
    p.o_l = static_cast<__nv_bfloat16 *>(o_l);
    p.lse = lse;
    if ((o_fg || o_l || lse) && !(o_fg && o_l && lse)) return cudaErrorInvalidValue;
    if (n_mirrors < 0 || n_mirrors > kMaxMirrors || (n_mirrors > 0 && !mirrors)) return cudaErrorInvalidValue;
    p.n_mirror = n_mirrors;
    for (int i = 0; i < kMaxMirrors; ++i) p.mirror[i] = i < n_mirrors ? static_cast<__nv_bfloat16 *>(mirrors[i]) : nullptr;
    p.n_tokens = pb.n_tokens;
    p.m = (int)pb.m;
    p.n = (int)pb.top_n;
    p.w = (int)pb.window;
    p.R = (int)(pb.block_size / BK);
    p.logR = 0;
    while ((1 << p.logR) < p.R) ++p.logR;
    if ((1 << p.logR) != p.R) return cudaErrorNotSupported;   // blocks of 64 * 2^k tokens
    p.tiles = pb.n_tokens / BK;
    p.total_blocks = pb.slabs * p.tiles;
    p.scale_log2 = pb.scale * 1.4426950408889634f;
    p.withhold_v_step = pb.withhold_v_step;
    const int sms = sm_count();
    if (sms <= 0) return cudaErrorInvalidDevice;
    const int64_t want = (p.total_blocks + NSLOT - 1) / NSLOT;
    const int grid = (int)(want < sms ? want : sms);
    if (p.o_fg && n_mirrors > 0) return cudaErrorInvalidValue;   // one extra output kind per launch
    const int mode = p.o_fg ? 1 : (n_mirrors > 0 ? 2 : 0);
    switch (p.logR * 3 + mode) {
        case 0: return launch_kernel<0, 0>(tq, tk, tv, p, grid, stream);
        case 1: return launch_kernel<0, 1>(tq, tk, tv, p, grid, stream);
        case 2: return launch_kernel<0, 2>(tq, tk, tv, p, grid, stream);
        case 6: return launch_kernel<2, 0>(tq, tk, tv, p, grid, stream);
        case 7: return launch_kernel<2, 1>(tq, tk, tv, p, grid, stream);
        case 8: return launch_kernel<2, 2>(tq, tk, tv, p, grid, stream);
        case 12: return launch_kernel<4, 0>(tq, tk, tv, p, grid, stream);
        case 13: return launch_kernel<4, 1>(tq, tk, tv, p, grid, stream);
        case 14: return launch_kernel<4, 2>(tq, tk, tv, p, grid, stream);
        default: return cudaErrorNotSupported;   // blocks of 64, 256 or 1024 tokens
    }
}

}  // namespace bsa

// Compressed branch (a) and top-n block selection of branch (b), BSA section
// of the MOSAIC note, on the sm_100a tensor cores with fp32-accurate products:
//
//   z_ij = s·q̄_i·k̄_j,   o_cg_i = Σ_j softmax_j(z_ij) v̄_j,
//   sel_i = top-n blocks j by (z_ij desc, j asc).
//
// Three-pass tf32: every fp32 operand x is split as x = x_hi + x_lo (x_hi = x
// with the 13 low mantissa bits cleared, an exact tf32 value; x_lo = x - x_hi,
// exact in fp32, of which the tensor core reads the tf32 part) and a product
// as a_hi·b_hi + a_hi·b_lo + a_lo·b_hi: three tcgen05.mma passes of kind tf32
// into one fp32 accumulator in TMEM. The dropped a_lo·b_lo term and the
// truncated low bits of the remainders leave a relative error below 2^-19 per
// product, so the logits that decide the ranking stay far inside its 1e-4
// margin. Each tile's P·V is a fresh accumulation (12 MMAs for each half of
// its keys, into the half's own TMEM columns); the tiles are summed in fp32
// registers.
//
// One CTA owns 128 query blocks (rows) of one slab and streams the slab's key
// blocks in tiles of 64 (the m×m logit matrix never leaves the SM):
//   warps 0-7  : two threads per row (TMEM lane): thread (q = warp%4, h = warp/4)
//                owns row 32q + lane and the keys 32h..32h+31 of each tile. It
//                reads those 32 logits, updates its own sorted top-n list and
//                online softmax, stores its half of P in tf32 parts for the
//                P·V MMA and folds its half's previous P·V into an fp32
//                accumulator. At the end half 1 hands its state to half 0
//                through tensor memory and half 0 merges both.
//   warps 8-11 : converters: read q̄, k̄, v̄ rows (fp32, L2-resident), split them
//                into tf32 parts and store them in the MMA's 128-byte-swizzled
//                K-major layout (V transposed: rows are features, keys run
//                along K); K runs one tile ahead of V
//   warp 12    : S warp (one elected lane issues): S(j) = Q·K(j)ᵀ into TMEM
//                buffer j%2
//   warp 13    : P·V warp (one elected lane issues): O_h(j) = P(j)[:, half h] ·
//                V(j)[half h, :] into TMEM buffer j%2, both halves. Two issuing
//                threads: one thread issues a tcgen05.mma about every 55-60
//                cycles at best, and a tile needs 48 of them
//   warps 14-15: complete the fourth warpgroup (registers are allocated by
//                whole warpgroups) and only give their registers away
// The row threads hold their logits, output row and top-n list in registers;
// a register split (setmaxnreg) moves registers to them from the other warps,
// by whole warpgroups.
// Given a workspace, a split kernel first writes every tile's tf32 parts, as
// the byte image of its shared-memory layout, once per slab; the converter
// warps then give way to one copy thread (bulk copies of those images), and no
// CTA re-splits the slab's key tiles.
// Every wait on an mbarrier is bounded (2 s); on expiry the CTA records a
// timeout (when given a status word), writes -1 as its rows' block indices,
// drains its MMAs and returns.
#include <math_constants.h>
#include <stddef.h>

#include "tc_common.cuh"

namespace bsa {
namespace {

using namespace tc;

constexpr int BM = 128;                    // query blocks per CTA
constexpr int BN = 64;                     // key blocks per tile
constexpr int D = 64;                      // head dim
constexpr int NTHREADS = 32 * 16;          // four whole warpgroups (see the register split)
constexpr int RROWS = 128 * 128;           // bytes of one 128-row swizzled region
constexpr int KROWS = 64 * 128;            // bytes of one 64-row swizzled region
constexpr uint32_t TMEM_COLS = 512;        // S buffers at 0 and 64; O(buffer b, half h) at 128 + 128b + 64h
// Register split: the CTA is launched with 128 registers a thread (512
// threads, one CTA per SM); the two row warpgroups rise to kRowRegs, the other
// two warpgroups drop to kCtlRegs. 256·kRowRegs + 256·kCtlRegs must not exceed
// 512·128 (the host checks the compiled launch count), or setmaxnreg.inc would
// wait forever.
constexpr int kRowRegs = 184, kCtlRegs = 72;
constexpr int kRegsNeeded = 256 * kRowRegs + 256 * kCtlRegs;

// instruction descriptor: D f32, A and B tf32, both K-major, M = 128, N = 64
constexpr uint32_t kIdesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(64 >> 3) << 17) |
                            ((uint32_t)(128 >> 4) << 24);

struct alignas(1024) Smem {
    uint8_t qhi[2][RROWS], qlo[2][RROWS];           // A of S: row x feature; region c: features 32c..32c+31
    uint8_t khi[2][2][KROWS], klo[2][2][KROWS];     // B of S, [stage][region]: key x feature
    uint8_t vhi[2][KROWS], vlo[2][KROWS];           // B of P·V, [region]: feature x key; region c: keys 32c..
    uint8_t phi[2][RROWS], plo[2][RROWS];           // A of P·V, [region]: row x key
    uint64_t q_full, k_full[2], k_empty[2], v_full, v_empty;
    uint64_t s_full[2], s_free[2], p_full, p_empty, o_full[2], o_free[2], drain, drain_pv;
    uint64_t merge[4];                              // [row quarter]: half 1's final state handed over
    uint32_t tmem_base;
    int abort_flag;
};

static_assert(sizeof(Smem) + 1024 <= 227 * 1024, "shared memory of one CTA");
// Split images (per slab): Q row tile rt at rt·QIMG (hi regions, then lo), key
// tile j of K and of V at j·KIMG (hi regions, then lo) in their own arrays.
constexpr int QIMG = 4 * RROWS, KIMG = 4 * KROWS;
static_assert(offsetof(Smem, qlo) == offsetof(Smem, qhi) + 2 * RROWS && offsetof(Smem, vlo) == offsetof(Smem, vhi) + 2 * KROWS,
              "hi and lo parts adjacent, as in the split images");

struct Args {
    const float *q, *k, *v;                // this slab's q̄, k̄, v̄ [m][64]
    const uint8_t *qimg, *kimg, *vimg;     // this slab's split images (workspace path), else null
    float *o_cg;                           // this slab's [m][64]
    int32_t *idx;                          // this slab's [m][n]
    float *lse;                            // this slab's [m] (training output), or null
    int m;
    float sl2;                             // s·log2(e)
    uint32_t *status;                      // nullable
};

// Split four fp32 values into a tf32 high part and the fp32 remainder; store
// them as one 16-byte chunk each.
__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }
__device__ __forceinline__ void store_split(uint8_t *hi, uint8_t *lo, uint32_t off, float4 x) {
    float4 h, l;
    h.x = tf32_hi(x.x);
    h.y = tf32_hi(x.y);
    h.z = tf32_hi(x.z);
    h.w = tf32_hi(x.w);
    // x - h, exact, two lanes per packed FMA
    const float2 l01 = __ffma2_rn(make_float2(h.x, h.y), make_float2(-1.f, -1.f), make_float2(x.x, x.y));
    const float2 l23 = __ffma2_rn(make_float2(h.z, h.w), make_float2(-1.f, -1.f), make_float2(x.z, x.w));
    l.x = l01.x;
    l.y = l01.y;
    l.z = l23.x;
    l.w = l23.y;
    *reinterpret_cast<float4 *>(hi + off) = h;
    *reinterpret_cast<float4 *>(lo + off) = l;
}

// Rows [row0, row0+NROWS) of a [m][64] fp32 matrix as a K-major operand: row
// r's features 32c..32c+31 in region c. Rows at or past m are zero.
// t: this thread's index among the 128 converters.
template <int NROWS>
__device__ __forceinline__ void convert_rows(const float *__restrict__ src, int row0, int m, int t, uint8_t *hi0,
                                             uint8_t *hi1, uint8_t *lo0, uint8_t *lo1) {
    constexpr int PER = NROWS * 16 / 128;  // float4 per thread
    float4 x[PER];
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int i = t + 128 * u, r = i >> 4, c4 = i & 15;
        x[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row0 + r < m) x[u] = __ldg(reinterpret_cast<const float4 *>(src + (int64_t)(row0 + r) * D) + c4);
    }
#pragma unroll
    for (int u = 0; u < PER; ++u) {
        const int i = t + 128 * u, r = i >> 4, c4 = i & 15;
        store_split(c4 < 8 ? hi0 : hi1, c4 < 8 ? lo0 : lo1, sw128_offset(r, c4 & 7), x[u]);
    }
}

// Keys [key0, key0+64) of v̄ [m][64], transposed into the K-major B operand of
// P·V: row f (feature) holds the 64 keys, region c keys 32c..32c+31. Each
// thread moves two 4x4 blocks (4 keys x 4 features). Keys past m are zero.
__device__ __forceinline__ void convert_v(const float *__restrict__ src, int key0, int m, int t, uint8_t *hi0,
                                          uint8_t *hi1, uint8_t *lo0, uint8_t *lo1) {
    float4 x[2][4];
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const int blk = t + 128 * b, kg = blk & 15, fg = blk >> 4;   // key group fastest: conflict-free stores
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int key = key0 + 4 * kg + a;
            x[b][a] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (key < m) x[b][a] = __ldg(reinterpret_cast<const float4 *>(src + (int64_t)key * D) + fg);
        }
    }
#pragma unroll
    for (int b = 0; b < 2; ++b) {
        const int blk = t + 128 * b, kg = blk & 15, fg = blk >> 4;
        uint8_t *hi = kg < 8 ? hi0 : hi1, *lo = kg < 8 ? lo0 : lo1;
        store_split(hi, lo, sw128_offset(4 * fg + 0, kg & 7), make_float4(x[b][0].x, x[b][1].x, x[b][2].x, x[b][3].x));
        store_split(hi, lo, sw128_offset(4 * fg + 1, kg & 7), make_float4(x[b][0].y, x[b][1].y, x[b][2].y, x[b][3].y));
        store_split(hi, lo, sw128_offset(4 * fg + 2, kg & 7), make_float4(x[b][0].z, x[b][1].z, x[b][2].z, x[b][3].z));
        store_split(hi, lo, sw128_offset(4 * fg + 3, kg & 7), make_float4(x[b][0].w, x[b][1].w, x[b][2].w, x[b][3].w));
    }
}

__device__ void convert_role(const Args &a, Smem &sh, int t, int row0, int T, volatile int *abort_flag) {
    auto wait_c = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_try_wait(b, par) || wait_bar(b, par, abort_flag, a.status));
    };
    auto make_k = [&](int x) -> bool {     // K(x) into stage x%2 once S(x-2) has read it
        const int st = x & 1;
        if (!wait_c(&sh.k_empty[st], ((x >> 1) & 1) ^ 1)) return false;
        convert_rows<BN>(a.k, x * BN, a.m, t, sh.khi[st][0], sh.khi[st][1], sh.klo[st][0], sh.klo[st][1]);
        fence_proxy_async();
        mbar_arrive(&sh.k_full[st]);
        return true;
    };
    for (int h = 0; h < BM; h += 64)       // Q in two halves of 64 rows (fewer registers)
        convert_rows<64>(a.q, row0 + h, a.m, t, sh.qhi[0] + h * 128, sh.qhi[1] + h * 128, sh.qlo[0] + h * 128,
                         sh.qlo[1] + h * 128);
    fence_proxy_async();
    mbar_arrive(&sh.q_full);
    if (!make_k(0)) return;
    for (int j = 0; j < T; ++j) {
        if (j + 1 < T && !make_k(j + 1)) return;
        // V(j) once P·V(j-1) has read the single V buffer
        if (!wait_c(&sh.v_empty, (j & 1) ^ 1)) return;
        convert_v(a.v, j * BN, a.m, t, sh.vhi[0], sh.vhi[1], sh.vlo[0], sh.vlo[1]);
        fence_proxy_async();
        mbar_arrive(&sh.v_full);
    }
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) completing on `bar`.
__device__ __forceinline__ void bulk_copy(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// Workspace path: one thread copies the split images in the converters'
// order (Q; K(0); per tile j, K(j+1) and V(j)).
__device__ void copy_role(const Args &a, Smem &sh, int row0, int T, volatile int *abort_flag) {
    // most recent copy of each kind (for the drain on abort): K stage and parity, V parity
    bool q_issued = false;
    int last_kst = -1, last_vpar = -1;
    uint32_t last_kpar = 0;
    auto wait_c = [&](uint64_t *b, uint32_t par) -> bool {
        return mbar_try_wait(b, par) || wait_bar(b, par, abort_flag, a.status);
    };
    auto copy_k = [&](int x) -> bool {      // K(x) into stage x%2 once S(x-2) has read it
        const int st = x & 1;
        if (!wait_c(&sh.k_empty[st], ((x >> 1) & 1) ^ 1)) return false;
        mbar_expect_tx(&sh.k_full[st], KIMG);
        bulk_copy(sh.khi[st][0], a.kimg + (int64_t)x * KIMG, 2 * KROWS, &sh.k_full[st]);
        bulk_copy(sh.klo[st][0], a.kimg + (int64_t)x * KIMG + 2 * KROWS, 2 * KROWS, &sh.k_full[st]);
        last_kst = st;
        last_kpar = (x >> 1) & 1;
        return true;
    };
    bool ok = true;
    mbar_expect_tx(&sh.q_full, QIMG);
    bulk_copy(sh.qhi[0], a.qimg + (int64_t)(row0 / BM) * QIMG, QIMG, &sh.q_full);
    q_issued = true;
    ok = copy_k(0);
    for (int j = 0; ok && j < T; ++j) {
        if (j + 1 < T && !(ok = copy_k(j + 1))) break;
        if (!(ok = wait_c(&sh.v_empty, (j & 1) ^ 1))) break;
        mbar_expect_tx(&sh.v_full, KIMG);
        bulk_copy(sh.vhi[0], a.vimg + (int64_t)j * KIMG, KIMG, &sh.v_full);
        last_vpar = j & 1;
    }
    if (!ok) {                              // let the copies in flight land before the CTA exits
        if (q_issued) drain_bar(&sh.q_full, 0);
        if (last_kst >= 0) {
            drain_bar(&sh.k_full[last_kst], last_kpar);
            drain_bar(&sh.k_full[last_kst ^ 1], last_kpar ^ (last_kst == 0 ? 1u : 0u));
        }
        if (last_vpar >= 0) drain_bar(&sh.v_full, (uint32_t)last_vpar);
    }
}

// D = A·Bᵀ in three tf32 passes (hi·hi, hi·lo, lo·hi) over K = 64: 24 MMAs.
// a*/b*: the two 32-wide K regions of each operand's parts.
__device__ __forceinline__ void mma_3pass(uint32_t d, const uint8_t *ah0, const uint8_t *ah1, const uint8_t *al0,
                                          const uint8_t *al1, const uint8_t *bh0, const uint8_t *bh1,
                                          const uint8_t *bl0, const uint8_t *bl1) {
    const uint64_t ah[2] = {desc_kmajor_sw128(ah0), desc_kmajor_sw128(ah1)};
    const uint64_t al[2] = {desc_kmajor_sw128(al0), desc_kmajor_sw128(al1)};
    const uint64_t bh[2] = {desc_kmajor_sw128(bh0), desc_kmajor_sw128(bh1)};
    const uint64_t bl[2] = {desc_kmajor_sw128(bl0), desc_kmajor_sw128(bl1)};
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)          // 8 tf32 (32 B) per MMA
        mma_tf32(d, ah[kk >> 2] + 2 * (kk & 3), bh[kk >> 2] + 2 * (kk & 3), kIdesc, kk > 0);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_tf32(d, ah[kk >> 2] + 2 * (kk & 3), bl[kk >> 2] + 2 * (kk & 3), kIdesc, 1u);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
        mma_tf32(d, al[kk >> 2] + 2 * (kk & 3), bh[kk >> 2] + 2 * (kk & 3), kIdesc, 1u);
}

// S(j) = Q·K(j)ᵀ into TMEM buffer j%2, for every key tile j.
// D = A·Bᵀ in three tf32 passes over K = 32 (one 128-byte region of each operand): 12 MMAs.
__device__ __forceinline__ void mma_3pass_k32(uint32_t d, const uint8_t *ah0, const uint8_t *al0, const uint8_t *bh0,
                                              const uint8_t *bl0) {
    const uint64_t ah = desc_kmajor_sw128(ah0), al = desc_kmajor_sw128(al0);
    const uint64_t bh = desc_kmajor_sw128(bh0), bl = desc_kmajor_sw128(bl0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) mma_tf32(d, ah + 2 * kk, bh + 2 * kk, kIdesc, kk > 0);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) mma_tf32(d, ah + 2 * kk, bl + 2 * kk, kIdesc, 1u);
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) mma_tf32(d, al + 2 * kk, bh + 2 * kk, kIdesc, 1u);
}

__device__ void mma_s_role(const Args &a, Smem &sh, uint32_t tmem, int T, volatile int *abort_flag) {
    const bool leader = elect_one();
    auto wait_w = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_try_wait(b, par) || wait_bar(b, par, abort_flag, a.status));
    };
    bool ok = wait_w(&sh.q_full, 0);
    for (int j = 0; ok && j < T; ++j) {
        const int st = j & 1;
        if (!(ok = wait_w(&sh.k_full[st], (j >> 1) & 1))) break;
        if (!(ok = wait_w(&sh.s_free[st], ((j >> 1) & 1) ^ 1))) break;
        fence_after();
        if (leader) {
            mma_3pass(tmem + 64 * st, sh.qhi[0], sh.qhi[1], sh.qlo[0], sh.qlo[1], sh.khi[st][0], sh.khi[st][1],
                      sh.klo[st][0], sh.klo[st][1]);
            commit(&sh.s_full[st]);
            commit(&sh.k_empty[st]);
        }
        __syncwarp();
    }
    // every MMA this thread issued must be complete before TMEM is freed
    if (leader) commit(&sh.drain);
    __syncwarp();
    drain_bar(&sh.drain, 0);
}

// O(i) = P(i)·V(i) into TMEM buffer i%2, for every key tile i.
__device__ void mma_pv_role(const Args &a, Smem &sh, uint32_t tmem, int T, volatile int *abort_flag) {
    const bool leader = elect_one();
    auto wait_w = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_try_wait(b, par) || wait_bar(b, par, abort_flag, a.status));
    };
    bool ok = true;
    for (int i = 0; ok && i < T; ++i) {
        if (!(ok = wait_w(&sh.p_full, i & 1) && wait_w(&sh.v_full, i & 1) &&
                   wait_w(&sh.o_free[i & 1], ((i >> 1) & 1) ^ 1)))
            break;
        fence_after();
        if (leader) {
            // O_h(i) = P(i)[:, keys of half h] · V(i)[keys of half h, :]: K = 32 from region h
#pragma unroll
            for (int hh = 0; hh < 2; ++hh)
                mma_3pass_k32(tmem + 128 + 128 * (i & 1) + 64 * hh, sh.phi[hh], sh.plo[hh], sh.vhi[hh], sh.vlo[hh]);
            commit(&sh.o_full[i & 1]);
            commit(&sh.v_empty);
            commit(&sh.p_empty);
        }
        __syncwarp();
    }
    if (leader) commit(&sh.drain_pv);
    __syncwarp();
    drain_bar(&sh.drain_pv, 0);
}

// lv/li = the first NSEL entries of s (keys 0..NSEL-1) sorted by (value
// descending, key ascending): a bitonic network on registers.
template <int NSEL>
__device__ __forceinline__ void sort_desc(const float *s, float *lv, int *li) {
#pragma unroll
    for (int p = 0; p < NSEL; ++p) {
        lv[p] = s[p];
        li[p] = p;
    }
#pragma unroll
    for (int k = 2; k <= NSEL; k <<= 1)
#pragma unroll
        for (int jj = k >> 1; jj > 0; jj >>= 1)
#pragma unroll
            for (int p = 0; p < NSEL; ++p) {
                const int q = p ^ jj;
                if (q <= p) continue;
                // (p, q) in descending order within ascending-k blocks of alternating direction
                const bool desc = (p & k) == 0;
                const bool q_above = lv[q] > lv[p] || (lv[q] == lv[p] && li[q] < li[p]);
                if (q_above == desc) {
                    const float tv = lv[p];
                    lv[p] = lv[q];
                    lv[q] = tv;
                    const int ti = li[p];
                    li[p] = li[q];
                    li[q] = ti;
                }
            }
}

// Insert (v, j) into the descending list lv/li of NSEL entries. Keys arrive in
// ascending j, so an equal logit already in the list keeps its place: the
// strict comparison realises the (z desc, j asc) order.
template <int NSEL>
__device__ __forceinline__ void list_insert(float *lv, int *li, float v, int j) {
#pragma unroll
    for (int p = NSEL - 1; p > 0; --p) {
        const bool up = v > lv[p - 1], here = v > lv[p];
        const float nv = up ? lv[p - 1] : (here ? v : lv[p]);
        const int ni = up ? li[p - 1] : (here ? j : li[p]);
        lv[p] = nv;
        li[p] = ni;
    }
    if (v > lv[0]) {
        lv[0] = v;
        li[0] = j;
    }
}

// 32 lanes x 16 columns: thread t of the warp reads / writes TMEM lane (base + t), columns [col, col+16).
__device__ __forceinline__ void tmem_ld16c(uint32_t taddr, float *r) {
    uint32_t *u = reinterpret_cast<uint32_t *>(r);
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(u[0]), "=r"(u[1]), "=r"(u[2]), "=r"(u[3]), "=r"(u[4]), "=r"(u[5]), "=r"(u[6]), "=r"(u[7]),
          "=r"(u[8]), "=r"(u[9]), "=r"(u[10]), "=r"(u[11]), "=r"(u[12]), "=r"(u[13]), "=r"(u[14]), "=r"(u[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16c(uint32_t taddr, const float *r) {
    const uint32_t *u = reinterpret_cast<const uint32_t *>(r);
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(u[0]), "r"(u[1]), "r"(u[2]), "r"(u[3]), "r"(u[4]), "r"(u[5]), "r"(u[6]), "r"(u[7]), "r"(u[8]),
        "r"(u[9]), "r"(u[10]), "r"(u[11]), "r"(u[12]), "r"(u[13]), "r"(u[14]), "r"(u[15])
        : "memory");
}

// (v, i) ranks before (w, k) in the selection order (logit descending, block index ascending)
__device__ __forceinline__ bool ranks_before(float v, int i, float w, int k) { return v > w || (v == w && i < k); }

// Row threads: two per row. Thread (q, h, lane) owns row r = 32q + lane (TMEM lane) and, of
// every key tile, the 32 keys 32h..32h+31: their logits, its own sorted top-n list of those keys,
// its own online softmax (running max and sum) and its own P·V accumulator O_h over them. The
// two halves never exchange anything per tile; at the end half 1 hands its state to half 0
// through tensor memory and half 0 merges: the lists by the selection order, the softmax states
// by rescaling both to the larger maximum.
template <int NSEL>
__device__ void row_role(const Args &a, Smem &sh, uint32_t tmem, int q, int h, int lane, int row0, int T,
                         volatile int *abort_flag) {
    const int r = 32 * q + lane;           // row of the tile = TMEM lane
    const int row = row0 + r;
    const uint32_t tl = (uint32_t)(32 * q) << 16;
    constexpr int HK = BN / 2;             // keys of a tile per thread
    auto wait_s = [&](uint64_t *b, uint32_t par) -> bool {
        return __all_sync(0xffffffffu, mbar_try_wait(b, par) || wait_bar(b, par, abort_flag, a.status));
    };
    float lv[NSEL];
    int li[NSEL];
#pragma unroll
    for (int p = 0; p < NSEL; ++p) {
        lv[p] = -CUDART_INF_F;
        li[p] = 0x7fffffff;
    }
    float m_run = -CUDART_INF_F, l_run = 0.f;   // log2-domain running max and sum of this half-row
    float m_acc = -CUDART_INF_F;                // max that o is expressed against
    float m_even = -CUDART_INF_F, m_odd = -CUDART_INF_F;   // the max P(j) was formed against, j even / odd
    float o[D];
#pragma unroll
    for (int c = 0; c < D; ++c) o[c] = 0.f;
    auto fold_o = [&](int i) -> bool {     // o += O_h(i), rescaled to the newer max
        if (!wait_s(&sh.o_full[i & 1], (i >> 1) & 1)) return false;
        fence_after();
        const uint32_t to = tmem + 128 + 128 * (i & 1) + 64 * h + tl;
        const float m_i = (i & 1) ? m_odd : m_even;
        // (a half-row with no valid key yet has m = -inf and o = 0)
        const float f = m_acc == -CUDART_INF_F ? 0.f : ex2(m_acc - m_i);
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {   // 32 columns at a time (registers)
            float part[32];
            tmem_ld32(to + 32 * hh, part);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < 16; ++c) {
                const float2 r2 = __ffma2_rn(make_float2(o[32 * hh + 2 * c], o[32 * hh + 2 * c + 1]), make_float2(f, f),
                                             make_float2(part[2 * c], part[2 * c + 1]));
                o[32 * hh + 2 * c] = r2.x;
                o[32 * hh + 2 * c + 1] = r2.y;
            }
        }
        fence_before();
        mbar_arrive(&sh.o_free[i & 1]);
        m_acc = m_i;
        return true;
    };
    bool ok = true;
    for (int j = 0; j < T; ++j) {
        const int st = j & 1;
        if (!(ok = wait_s(&sh.s_full[st], (j >> 1) & 1))) break;
        fence_after();
        float s[HK];                       // raw logits q̄·k̄ of keys j*64 + 32h .. +31
        tmem_ld32(tmem + 64 * st + 32 * h + tl, s);
        tmem_wait_ld();
        fence_before();
        mbar_arrive(&sh.s_free[st]);
        const int key0 = j * BN + HK * h;
        if (key0 + HK > a.m) {
#pragma unroll
            for (int c = 0; c < HK; ++c)
                if (key0 + c >= a.m) s[c] = -CUDART_INF_F;
        }
        // ---- top-n of this half's keys: candidates beat the list's n-th entry; taken in key
        //      order. The first tile seeds the list with its first NSEL logits, sorted.
        int g0 = 0;
        if (j == 0) {
            sort_desc<NSEL>(s, lv, li);
#pragma unroll
            for (int p = 0; p < NSEL; ++p) li[p] += key0;
            g0 = NSEL / 8;
        }
        float gm[HK / 8];                  // maxima of the 4 groups of 8 logits
#pragma unroll
        for (int g = 0; g < HK / 8; ++g)
            gm[g] = fmax3(fmax3(s[8 * g], s[8 * g + 1], s[8 * g + 2]), fmax3(s[8 * g + 3], s[8 * g + 4], s[8 * g + 5]),
                          fmaxf(s[8 * g + 6], s[8 * g + 7]));
#pragma unroll
        for (int g = 0; g < HK / 8; ++g) {
            if (g < g0) continue;
            const float thr = lv[NSEL - 1];
            if (!(gm[g] > thr)) continue;  // no candidate in this group
            uint32_t cand = 0;
#pragma unroll
            for (int u = 0; u < 8; ++u)
                if (s[8 * g + u] > thr) cand |= 1u << u;
            while (cand) {
                const int u = __ffs(cand) - 1;
                cand &= cand - 1;
                float v = s[8 * g];
#pragma unroll
                for (int uu = 1; uu < 8; ++uu)
                    if (u == uu) v = s[8 * g + uu];
                if (v > lv[NSEL - 1]) list_insert<NSEL>(lv, li, v, key0 + 8 * g + u);
            }
        }
        // ---- online softmax (log2 domain) of the half-row
        const float mt = fmaxf(fmaxf(gm[0], gm[1]), fmaxf(gm[2], gm[3]));
        const float m_new = fmaxf(m_run, mt * a.sl2);
        const float m_sub = m_new == -CUDART_INF_F ? 0.f : m_new;   // no valid key yet: P = 0
        // exponents, then all exponentials, then four packed partial sums: in-order issue
        // never waits on one exp-unit result while later independent ones could be queued
        float ls;
        {
            const float2 sc2 = make_float2(a.sl2, a.sl2), nm2 = make_float2(-m_sub, -m_sub);
#pragma unroll
            for (int c = 0; c < HK / 2; ++c) {
                const float2 x = __ffma2_rn(make_float2(s[2 * c], s[2 * c + 1]), sc2, nm2);
                s[2 * c] = x.x;
                s[2 * c + 1] = x.y;
            }
#pragma unroll
            for (int c = 0; c < HK; ++c) s[c] = ex2(s[c]);
            float2 acc4[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                              make_float2(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < HK / 2; ++c) acc4[c & 3] = __fadd2_rn(acc4[c & 3], make_float2(s[2 * c], s[2 * c + 1]));
            const float2 t2 = __fadd2_rn(__fadd2_rn(acc4[0], acc4[1]), __fadd2_rn(acc4[2], acc4[3]));
            ls = t2.x + t2.y;
        }
        l_run = (m_run == -CUDART_INF_F ? 0.f : l_run * ex2(m_run - m_new)) + ls;
        m_run = m_new;
        if (st) m_odd = m_new;
        else m_even = m_new;
        // ---- P(j) of this half in tf32 parts (region h of the P tile), once P·V(j-1) has read
        //      the single P buffer
        if (!(ok = wait_s(&sh.p_empty, (j & 1) ^ 1))) break;
#pragma unroll
        for (int c = 0; c < 8; ++c)
            store_split(sh.phi[h], sh.plo[h], sw128_offset(r, c),
                        make_float4(s[4 * c], s[4 * c + 1], s[4 * c + 2], s[4 * c + 3]));
        fence_proxy_async();
        mbar_arrive(&sh.p_full);
        if (j > 0 && !(ok = fold_o(j - 1))) break;
    }
    if (ok && T > 0) ok = fold_o(T - 1);
    // ---- half 1 hands (o, list, m, l) to half 0 through tensor memory: columns 384..447 (o),
    //      448.. (list values), 480.. (list indices), 192 (m, l: half 1's own, now idle, O columns)
    constexpr uint32_t kXO = 384, kXV = 448, kXI = 480, kXML = 192;
    if (h == 1) {
        if (ok) {
            tmem_st32(tmem + kXO + tl, o);
            tmem_st32(tmem + kXO + 32 + tl, o + 32);
#pragma unroll
            for (int c = 0; c < NSEL; c += 16) {
                float v16[16], i16[16];
#pragma unroll
                for (int p = 0; p < 16; ++p) {
                    v16[p] = lv[c + p];
                    i16[p] = __int_as_float(li[c + p]);
                }
                tmem_st16c(tmem + kXV + c + tl, v16);
                tmem_st16c(tmem + kXI + c + tl, i16);
            }
            float ml[16];
#pragma unroll
            for (int p = 0; p < 16; ++p) ml[p] = p == 0 ? m_run : (p == 1 ? l_run : 0.f);
            tmem_st16c(tmem + kXML + tl, ml);
            tmem_wait_st();
        }
        fence_before();
        mbar_arrive(&sh.merge[q]);         // (also when aborting: half 0 then sees the abort flag)
        return;
    }
    if (ok) ok = wait_s(&sh.merge[q], 0);
    const bool live = row < a.m;           // rows past m are computed but not stored
    int32_t *ix = a.idx + (int64_t)row * NSEL;
    if (!ok) {                             // aborted: flag the rows for the selection kernel
        if (live) {
#pragma unroll
            for (int p = 0; p < NSEL; ++p) ix[p] = -1;
        }
        return;
    }
    // the tensor-memory loads below are warp-collective (.sync.aligned): every lane of the warp
    // takes part, rows past m included, and only the global stores are skipped for those
    fence_after();
    float mb, lb;
    {
        float ml[16];
        tmem_ld16c(tmem + kXML + tl, ml);
        tmem_wait_ld();
        mb = ml[0];
        lb = ml[1];
    }
    // ---- the two lists: keep, position by position, the better of this list's p-th and the
    //      other's (NSEL-1-p)-th entry (a bitonic sequence holding the top NSEL of both), then sort
#pragma unroll
    for (int c = 0; c < NSEL; c += 16) {
        float v16[16], i16[16];             // the other list's entries NSEL-1-c-15 .. NSEL-1-c
        tmem_ld16c(tmem + kXV + (NSEL - 16 - c) + tl, v16);
        tmem_ld16c(tmem + kXI + (NSEL - 16 - c) + tl, i16);
        tmem_wait_ld();
#pragma unroll
        for (int pp = 0; pp < 16; ++pp) {
            const int p = c + pp;           // partner entry NSEL-1-p = (NSEL-16-c) + (15-pp)
            const float w = v16[15 - pp];
            const int k = __float_as_int(i16[15 - pp]);
            if (ranks_before(w, k, lv[p], li[p])) {
                lv[p] = w;
                li[p] = k;
            }
        }
    }
    // bitonic merge of the NSEL entries into the selection order
#pragma unroll
    for (int jj = NSEL / 2; jj > 0; jj >>= 1)
#pragma unroll
        for (int p = 0; p < NSEL; ++p) {
            const int pq = p ^ jj;
            if (pq <= p) continue;
            if (ranks_before(lv[pq], li[pq], lv[p], li[p])) {
                const float tv = lv[p];
                lv[p] = lv[pq];
                lv[pq] = tv;
                const int ti = li[p];
                li[p] = li[pq];
                li[pq] = ti;
            }
        }
    if (live) {
        int4 *idst = reinterpret_cast<int4 *>(ix);
#pragma unroll
        for (int p = 0; p < NSEL / 4; ++p) idst[p] = make_int4(li[4 * p], li[4 * p + 1], li[4 * p + 2], li[4 * p + 3]);
    }
    // ---- the softmax states: both halves rescaled to the larger maximum
    const float m = fmaxf(m_run, mb);
    const float fa = m_run == -CUDART_INF_F ? 0.f : ex2(m_run - m), fb = mb == -CUDART_INF_F ? 0.f : ex2(mb - m);
    const float l = l_run * fa + lb * fb;
    const float inv = 1.f / l;
    // training: natural-log log-sum-exp of the row's scaled logits
    if (live && a.lse) a.lse[row] = (m + log2f(l)) * 0.69314718055994531f;
    float4 *dst = reinterpret_cast<float4 *>(a.o_cg + (int64_t)row * D);
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
        float ob[32];
        tmem_ld32(tmem + kXO + 32 * hh + tl, ob);
        tmem_wait_ld();
        if (!live) continue;
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            const int e = 32 * hh + 4 * c;
            dst[8 * hh + c] = make_float4((o[e] * fa + ob[4 * c] * fb) * inv, (o[e + 1] * fa + ob[4 * c + 1] * fb) * inv,
                                          (o[e + 2] * fa + ob[4 * c + 2] * fb) * inv,
                                          (o[e + 3] * fa + ob[4 * c + 3] * fb) * inv);
        }
    }
}

template <int NSEL, bool PRE>
__global__ void __launch_bounds__(NTHREADS, 1)
compress_tc_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar, const float *__restrict__ vbar,
                   float *__restrict__ o_cg, int32_t *__restrict__ idx, int m, float sl2, uint32_t *status,
                   const uint8_t *__restrict__ images, float *__restrict__ lse) {
    extern __shared__ uint8_t smem_raw[];
    Smem &sh = *reinterpret_cast<Smem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t slab = blockIdx.y;
    const int row0 = blockIdx.x * BM;
    const int T = (m + BN - 1) / BN;
    Args a;
    a.q = qbar + slab * (int64_t)m * D;
    a.k = kbar + slab * (int64_t)m * D;
    a.v = vbar + slab * (int64_t)m * D;
    a.o_cg = o_cg + slab * (int64_t)m * D;
    a.idx = idx + slab * (int64_t)m * NSEL;
    a.lse = lse ? lse + slab * (int64_t)m : nullptr;
    a.m = m;
    a.sl2 = sl2;
    a.status = status;
    a.qimg = a.kimg = a.vimg = nullptr;
    if (PRE) {
        const int64_t qbytes = (int64_t)((m + BM - 1) / BM) * QIMG, kbytes = (int64_t)T * KIMG;
        a.qimg = images + slab * (qbytes + 2 * kbytes);
        a.kimg = a.qimg + qbytes;
        a.vimg = a.kimg + kbytes;
    }
    volatile int *abort_flag = &sh.abort_flag;
    constexpr uint32_t kFill = PRE ? 1u : 128u;   // arrivals that complete a Q/K/V tile

    if (threadIdx.x == 0) {
        sh.abort_flag = 0;
        mbar_init(&sh.q_full, kFill);
        mbar_init(&sh.v_full, kFill);
        mbar_init(&sh.v_empty, 1);
        mbar_init(&sh.p_full, 256);
        mbar_init(&sh.p_empty, 1);
        mbar_init(&sh.drain, 1);
        mbar_init(&sh.drain_pv, 1);
        for (int qq = 0; qq < 4; ++qq) mbar_init(&sh.merge[qq], 32);
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.k_full[b], kFill);
            mbar_init(&sh.k_empty[b], 1);
            mbar_init(&sh.s_full[b], 1);
            mbar_init(&sh.s_free[b], 256);
            mbar_init(&sh.o_full[b], 1);
            mbar_init(&sh.o_free[b], 256);
        }
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 12) {
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

    if (warp < 8) {
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRowRegs));
        row_role<NSEL>(a, sh, tmem, warp & 3, warp >> 2, lane, row0, T, abort_flag);
    } else {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kCtlRegs));
        if (PRE) {
            if (warp == 8 && lane == 0) copy_role(a, sh, row0, T, abort_flag);
        } else if (warp < 12) {
            convert_role(a, sh, threadIdx.x - 256, row0, T, abort_flag);
        }
        if (warp == 12)
            mma_s_role(a, sh, tmem, T, abort_flag);
        else if (warp == 13)
            mma_pv_role(a, sh, tmem, T, abort_flag);
    }
    __syncwarp();

    fence_before();
    __syncthreads();
    if (warp == 12) {
        fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS)
                     : "memory");
    }
}

// The split images of one slab: CTA (c, slab) handles block rows 64c..64c+63
// (zero past m): their Q rows, and, if they form a key tile, that tile's K
// and transposed V (same layouts as the converters write to shared memory).
__global__ void __launch_bounds__(256)
split_images_kernel(const float *__restrict__ qbar, const float *__restrict__ kbar, const float *__restrict__ vbar,
                    uint8_t *__restrict__ images, int m) {
    const int64_t slab = blockIdx.y;
    const int r0 = blockIdx.x * 64, t = threadIdx.x;
    const int T = (m + BN - 1) / BN;
    const int64_t qbytes = (int64_t)((m + BM - 1) / BM) * QIMG, kbytes = (int64_t)T * KIMG;
    uint8_t *qimg = images + slab * (qbytes + 2 * kbytes);
    uint8_t *kimg = qimg + qbytes, *vimg = kimg + kbytes;
    const float *q = qbar + slab * (int64_t)m * D, *k = kbar + slab * (int64_t)m * D, *v = vbar + slab * (int64_t)m * D;
    // Q: rows r0.. are rows (r0 % 128).. of row tile r0 / 128
    {
        uint8_t *base = qimg + (int64_t)(r0 / BM) * QIMG + (r0 % BM) * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = t + 256 * u, r = i >> 4, c4 = i & 15;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r0 + r < m) x = __ldg(reinterpret_cast<const float4 *>(q + (int64_t)(r0 + r) * D) + c4);
            const int reg = c4 >> 3;
            store_split(base + reg * RROWS, base + 2 * RROWS + reg * RROWS, sw128_offset(r, c4 & 7), x);
        }
    }
    if (r0 >= T * BN) return;
    const int kt = r0 / BN;
    {
        uint8_t *base = kimg + (int64_t)kt * KIMG;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const int i = t + 256 * u, r = i >> 4, c4 = i & 15;
            float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
            if (r0 + r < m) x = __ldg(reinterpret_cast<const float4 *>(k + (int64_t)(r0 + r) * D) + c4);
            const int reg = c4 >> 3;
            store_split(base + reg * KROWS, base + 2 * KROWS + reg * KROWS, sw128_offset(r, c4 & 7), x);
        }
    }
    {
        uint8_t *base = vimg + (int64_t)kt * KIMG;
        const int kg = t & 15, fg = t >> 4;    // one 4x4 block per thread
        float4 x[4];
#pragma unroll
        for (int a2 = 0; a2 < 4; ++a2) {
            const int key = r0 + 4 * kg + a2;
            x[a2] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (key < m) x[a2] = __ldg(reinterpret_cast<const float4 *>(v + (int64_t)key * D) + fg);
        }
        uint8_t *hi = base + (kg >> 3) * KROWS, *lo = base + 2 * KROWS + (kg >> 3) * KROWS;
        store_split(hi, lo, sw128_offset(4 * fg + 0, kg & 7), make_float4(x[0].x, x[1].x, x[2].x, x[3].x));
        store_split(hi, lo, sw128_offset(4 * fg + 1, kg & 7), make_float4(x[0].y, x[1].y, x[2].y, x[3].y));
        store_split(hi, lo, sw128_offset(4 * fg + 2, kg & 7), make_float4(x[0].z, x[1].z, x[2].z, x[3].z));
        store_split(hi, lo, sw128_offset(4 * fg + 3, kg & 7), make_float4(x[0].w, x[1].w, x[2].w, x[3].w));
    }
}

template <int NSEL, bool PRE>
cudaError_t launch_tc_n(const Problem &p, const float *qbar, const float *kbar, const float *vbar, float *o_cg,
                        int32_t *idx, uint32_t *status, const uint8_t *images, cudaStream_t stream, float *lse) {
    const size_t smem = sizeof(Smem) + 1024;
    cudaError_t e = cudaFuncSetAttribute(compress_tc_kernel<NSEL, PRE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    // the register split must fit the registers the CTA is launched with
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, compress_tc_kernel<NSEL, PRE>);
    if (e != cudaSuccess) return e;
    if ((int64_t)fa.numRegs * NTHREADS < kRegsNeeded || fa.maxThreadsPerBlock < NTHREADS)
        return cudaErrorInvalidConfiguration;
    const dim3 grid((unsigned)((p.m + BM - 1) / BM), (unsigned)p.slabs);
    compress_tc_kernel<NSEL, PRE><<<grid, NTHREADS, smem, stream>>>(qbar, kbar, vbar, o_cg, idx, (int)p.m,
                                                                     p.scale * 1.4426950408889634f, status, images,
                                                                     lse);
    return cudaGetLastError();
}

template <bool PRE>
cudaError_t launch_tc(const Problem &p, const float *qbar, const float *kbar, const float *vbar, float *o_cg,
                      int32_t *idx, uint32_t *status, const uint8_t *images, cudaStream_t stream, float *lse) {
    if (p.top_n == 32)
        return launch_tc_n<32, PRE>(p, qbar, kbar, vbar, o_cg, idx, status, images, stream, lse);
    return launch_tc_n<16, PRE>(p, qbar, kbar, vbar, o_cg, idx, status, images, stream, lse);
}

}  // namespace

bool compress_tc_supported(const Problem &p) {
    return p.head_dim == D && (p.top_n == 16 || p.top_n == 32) && p.m <= 0x7fffffffLL / D;
}

size_t compress_tc_workspace_bytes(const Problem &p) {
    if (!compress_tc_supported(p)) return 0;
    const size_t rt = (size_t)((p.m + BM - 1) / BM), kt = (size_t)((p.m + BN - 1) / BN);
    return (size_t)p.slabs * (rt * QIMG + 2 * kt * KIMG);
}

cudaError_t launch_compress_tc(const Problem &p, const float *qbar, const float *kbar, const float *vbar,
                               float *o_cg, int32_t *idx, uint32_t *status, void *images, cudaStream_t stream,
                               float *lse) {
    if (!compress_tc_supported(p)) return cudaErrorNotSupported;
    if (!images) return launch_tc<false>(p, qbar, kbar, vbar, o_cg, idx, status, nullptr, stream, lse);
    const dim3 sgrid((unsigned)((p.m + BM - 1) / BM * 2), (unsigned)p.slabs);
    split_images_kernel<<<sgrid, 256, 0, stream>>>(qbar, kbar, vbar, static_cast<uint8_t *>(images), (int)p.m);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    return launch_tc<true>(p, qbar, kbar, vbar, o_cg, idx, status, static_cast<const uint8_t *>(images), stream,
                           lse);
}

}  // namespace bsa

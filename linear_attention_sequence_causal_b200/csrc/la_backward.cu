// Backward (training) pass of causal Taylor linear attention on the tensor cores.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED) §5 "Execution stages" names prefill during training; the
// forward is y_i = sum_{j<=i} a_ij v_j / den_i, a_ij = 1 + s_ij + s_ij^2/2,
// s_ij = q_i.k_j, den_i = sum_{j<=i} a_ij. For an upstream gradient dy:
//     g_i   = dy_i / den_i,   c_i = g_i . y_i,
//     ds_ij = (g_i . v_j - c_i) (1 + s_ij)         (j <= i, else 0),
//     dq_i  = sum_j ds_ij k_j,   dk_j = sum_i ds_ij q_i,   dv_j = sum_i a_ij g_i.
// Two persistent kernels, each one CTA per SM walking 128-row units longest
// first and sweeping the 128-row tiles of the other side:
//   DQ   unit = query tile: S = Q K^T (M=128 N=128 K=d'), X' = dY V^T (K=dv);
//        with c'_i = dy_i . y_i, ds'_ij = (X'_ij - c'_i)(1 + s_ij) (= den_i ds_ij),
//        bf16 in TMEM; dQ' += dS' K (A operand in TMEM, K as an MN-major
//        operand); den_i accumulates as the masked row sums of A. At the end
//        dq = dQ' / den, and G = dy / den (bf16) and c = g . y go to the
//        workspace (rows padded to a multiple of 128 with zeros);
//   DKV  unit = key tile: S^T = K Q^T, X^T = V G^T; A^T and dS^T in TMEM;
//        dV += A^T G and dK += dS^T Q (G and Q as MN-major operands).
// Each d'-wide tile (Q, K) sits in shared memory under the swizzle of its row
// width and serves both as a K-major operand (rows = M or N) and, read along
// its rows, as an MN-major operand (rows = K); each dv-wide tile (V, dY, G) sits in
// 64-column blocks under the 128-byte swizzle and serves both ways likewise.
// Roles (640 threads): warp 0 lane 0 loads by TMA (the unit's own tile(s) and a
// ring of the other side's tiles); warp 1 allocates TMEM and lane 0 issues S and
// X; lane 0 of warps 2 and 3 issue the products (dV or dQ; dK); warps 4-19
// (thread = TMEM lane x 32-column group) form A / dS and write the unit's
// results. Every hand-off is an mbarrier; every wait is bounded.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma_host.h"

namespace based {
namespace {

using namespace tc;

constexpr int C = 128;
constexpr int kRowGroups = 4;                        // row warps per TMEM lane quadrant
constexpr int kRowThreads = 128 * kRowGroups;        // thread = (row, 32-column group)
constexpr int kBwdThreads = 128 + kRowThreads;      // 4 control warps + the row warps
enum { MODE_DQ = 1, MODE_DKV = 2 };

template <int DF, int DV, int MODE>
struct BwdLayout {
    static constexpr int QK_SWIZZLE = DF * 2;
    static constexpr uint32_t QK_BYTES = C * DF * 2;          // d'-wide tile: 128 rows of d' bf16
    static constexpr uint32_t QK_SBO = 8 * DF * 2;            // 8 rows
    static constexpr uint32_t V_BLOCK = C * 128;              // 64 columns x 128 rows, 128-byte swizzle
    static constexpr uint32_t V_BYTES = C * DV * 2;           // dv-wide tile
    static constexpr bool HAS_C = MODE == MODE_DKV;           // c of the stage's query tile
    static constexpr int STAGES = 4;                          // ring stages of the other side's tiles
    static constexpr int NPI = MODE == MODE_DQ ? 1 : 2;       // product issuers
    static constexpr uint32_t STAGE_BYTES = QK_BYTES + V_BYTES + (HAS_C ? 1024 : 0);
    static constexpr uint32_t OFF_A1 = 0;                     // own d'-wide tile
    static constexpr uint32_t OFF_A2 = OFF_A1 + QK_BYTES;     // own dv-wide tile
    static constexpr uint32_t OFF_RING = OFF_A2 + V_BYTES;
    static constexpr uint32_t OFF_B2 = QK_BYTES;              // within a stage
    static constexpr uint32_t OFF_CB = QK_BYTES + V_BYTES;
    static constexpr uint32_t OFF_BAR = OFF_RING + STAGES * STAGE_BYTES;
    static constexpr uint32_t OFF_RED = OFF_BAR + 256;        // DQ: [2][groups][128] partial den, then c
    static constexpr uint32_t RED_BYTES = 2 * kRowGroups * 128 * 4;
    static constexpr uint32_t SMEM_NEED = OFF_RED + 2 * RED_BYTES + 1024;   // + alignment slack
    // At least 116 KB, so that one CTA sits on an SM and owns all 512 TMEM columns.
    static constexpr uint32_t SMEM_BYTES = SMEM_NEED > 116 * 1024 ? SMEM_NEED : 116 * 1024;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(QK_BYTES % 1024 == 0 && V_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "tile alignment");
    // TMEM: S [0,128) and X [128,256) in fp32; the bf16 MMA operands formed from
    // them (dS for DQ; A^T and dS^T for DKV), 64 columns each, in a region of their
    // own where it fits (SEP), else over the S / X columns they came from (K step j
    // at column 16 j); then dV (DKV) and dQ / dK.
    static constexpr bool SEP = MODE == MODE_DQ || (MODE == MODE_DKV && DV == 64);
    static constexpr uint32_t COL_S = 0, COL_X = 128;
    static constexpr int NPB = MODE == MODE_DQ ? 2 : 1;                          // operand buffers
    static constexpr uint32_t COL_P = SEP ? 256 : COL_S;     // dS (DQ; buffer pb at + 64 pb) or A^T (DKV)
    static constexpr uint32_t COL_D = SEP ? (MODE == MODE_DKV ? 320 : 256) : COL_X;   // dS^T (DKV)
    static constexpr uint32_t KSTEP_COLS = SEP ? 8 : 16;                          // column pitch of K steps
    static constexpr uint32_t COL_ACC1 = SEP ? 384 : 256;                         // dV (DKV)
    static constexpr uint32_t COL_ACC2 = MODE == MODE_DKV ? COL_ACC1 + DV : 384;   // dK (DKV) or dQ
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_ACC2 + DF <= TMEM_COLS, "tensor memory");
    static constexpr uint32_t ID_SX = idesc_bf16_f32(128, C, false, false);      // S, X: both operands K-major
    static constexpr uint32_t ID_ACC1 = idesc_bf16_f32(128, DV, false, true);    // dV += A^T G
    static constexpr uint32_t ID_ACC2 = idesc_bf16_f32(128, DF, false, true);    // dQ += dS K, dK += dS^T Q
};

enum {
    BB_FULL0 = 0,             // [4] TMA: ring stage s landed
    BB_EMPTY0 = 4,            // [4] MMA commits: ring stage s read (S / X and the products)
    BB_OWNFULL = 8,           // TMA: the unit's own tiles landed
    BB_OWNFREE,               // MMA commit: the unit's own tiles no longer read
    BB_SF,                    // MMA commit: S and X of the step ready
    BB_SXFREE,                // row warps: S and X of the step read into registers
    BB_PF0,                   // [2] row warps: A / dS of the step written into operand buffer pb
    BB_AFREE10 = BB_PF0 + 2,  // [2] MMA commit: product issuer 1 (dV or dQ) read operand buffer pb
    BB_AFREE2 = BB_AFREE10 + 2,   // MMA commit: product issuer 2 (dK) read its operand
    BB_ACCF,                  // MMA commits: the unit's accumulators complete (one per product issuer)
    BB_ACCE,                  // row warps: accumulators read out
    BB_LSUM,                  // DQ row warps: partial den of the unit written
    BB_CSUM,                  // DQ row warps: partial c of the unit written
    BB_NUM
};

struct BwdCtx {
    uint32_t sbase;
    uint64_t* bars;
    void* red;                // DQ reduction scratch in shared memory
    volatile int* abort_flag;
    unsigned* status;
    int N, Npad, BH, nt, nunits;
};

__device__ __forceinline__ bool bwait(const BwdCtx& cx, int bar, uint32_t parity) {
    return mbar_wait(&cx.bars[bar], parity, cx.abort_flag, cx.status);
}

// Unit u: its own tile index, its head and its sweep of the other side's tiles
// [t0, t1]. DQ: query tile qt (longest first) against key tiles 0..qt;
// DKV: key tile kt (longest first) against query tiles kt..nt-1.
template <int MODE>
__device__ __forceinline__ void bwd_unit(const BwdCtx& cx, int u, int& own, int& bh, int& t0, int& t1) {
    bh = u % cx.BH;
    if constexpr (MODE == MODE_DKV) {
        own = u / cx.BH;
        t0 = own;
        t1 = cx.nt - 1;
    } else {
        own = cx.nt - 1 - u / cx.BH;
        t0 = 0;
        t1 = own;
    }
}

__device__ __forceinline__ void bwd_drain(const BwdCtx& cx, uint64_t* bar, uint32_t parity) {
    if (!*cx.abort_flag || bar == nullptr) return;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity) && global_ns() - t0 < kWaitLimitNs) {}
}

struct BwdMaps {
    const CUtensorMap* own1;   // d'-wide own tile (q for DQ, k for DKV)
    const CUtensorMap* own2;   // dv-wide own tile (dy for DQ, v for DKV)
    const CUtensorMap* ring1;  // d'-wide ring tile (k for DQ, q for DKV)
    const CUtensorMap* ring2;  // dv-wide ring tile (v for DQ, G for DKV)
};

// ------------------------------------------------------------------ TMA producer (warp 0, lane 0)
template <int DF, int DV, int MODE>
__device__ __forceinline__ void bwd_producer(const BwdCtx& cx, const BwdMaps& m, const float* __restrict__ cw) {
    using L = BwdLayout<DF, DV, MODE>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int own, bh, t0, t1;
        bwd_unit<MODE>(cx, u, own, bh, t0, t1);
        if (k_unit >= 1 && !bwait(cx, BB_OWNFREE, (k_unit - 1) & 1)) { bwd_drain(cx, last, lastp); return; }
        uint64_t* of = &cx.bars[BB_OWNFULL];
        mbar_expect_tx(of, L::QK_BYTES + L::V_BYTES);
        tma_load_3d(cx.sbase + L::OFF_A1, m.own1, of, 0, own * C, bh);
#pragma unroll
        for (int h = 0; h < DV / 64; ++h)
            tma_load_3d(cx.sbase + L::OFF_A2 + h * L::V_BLOCK, m.own2, of, 64 * h, own * C, bh);
        last = of;
        lastp = k_unit & 1;
        for (int t = t0; t <= t1; ++t, ++step) {
            const int s = step % L::STAGES;
            if (step >= L::STAGES && !bwait(cx, BB_EMPTY0 + s, (step / L::STAGES - 1) & 1)) {
                bwd_drain(cx, last, lastp);
                return;
            }
            uint64_t* full = &cx.bars[BB_FULL0 + s];
            const uint32_t st = cx.sbase + L::OFF_RING + s * L::STAGE_BYTES;
            mbar_expect_tx(full, L::QK_BYTES + L::V_BYTES + (L::HAS_C ? C * 4 : 0));
            tma_load_3d(st, m.ring1, full, 0, t * C, bh);
#pragma unroll
            for (int h = 0; h < DV / 64; ++h)
                tma_load_3d(st + L::OFF_B2 + h * L::V_BLOCK, m.ring2, full, 64 * h, t * C, bh);
            if constexpr (L::HAS_C) bulk_load(st + L::OFF_CB, cw + (size_t)bh * cx.Npad + t * C, C * 4, full);
            last = full;
            lastp = (step / L::STAGES) & 1;
        }
    }
    bwd_drain(cx, last, lastp);
}

// ------------------------------------------------------------------ MMA issuers
// One thread issues S and X per step (warp 1); one or two others issue the
// step's products once the row warps have formed their operands (warp 2: dV or
// dQ; warp 3: dK). The S / X issuer runs ahead of the products: it waits only
// until the row warps have read the S / X it is about to overwrite (or, where
// A / dS overlay S / X, until the products of the previous step have read
// them). Each issuer commits its own arrival on the ring stage's EMPTY barrier.

// S / X issuer (warp 1, lane 0).
template <int DF, int DV, int MODE>
__device__ __forceinline__ void bwd_issue_sx(const BwdCtx& cx, uint32_t tmem) {
    using L = BwdLayout<DF, DV, MODE>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    const uint32_t a1 = cx.sbase + L::OFF_A1, a2 = cx.sbase + L::OFF_A2;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int own, bh, t0, t1;
        bwd_unit<MODE>(cx, u, own, bh, t0, t1);
        for (int t = t0; t <= t1; ++t, ++step) {
            const int s = step % L::STAGES;
            bool ok = true;
            if constexpr (!L::SEP) {
                // In place: the previous step's products read these S / X columns.
                if (step >= 1) {
                    ok = bwait(cx, BB_AFREE10, (step - 1) & 1);
                    if (ok && L::NPI > 1) ok = bwait(cx, BB_AFREE2, (step - 1) & 1);
                }
            } else {
                if (step >= 1) ok = bwait(cx, BB_SXFREE, (step - 1) & 1);
            }
            ok = ok && bwait(cx, BB_FULL0 + s, (step / L::STAGES) & 1);
            if (ok && t == t0) ok = bwait(cx, BB_OWNFULL, k_unit & 1);
            if (!ok) { bwd_drain(cx, last, lastp); return; }
            tc_fence_after();
            const uint32_t st = cx.sbase + L::OFF_RING + s * L::STAGE_BYTES;
            // S = own1 ring1^T (K = d'), both K-major.
#pragma unroll
            for (int j = 0; j < DF / 16; ++j)
                mma_bf16(tmem + L::COL_S, smem_desc_swizzled(a1, 16, L::QK_SBO, L::QK_SWIZZLE) + 2 * j,
                         smem_desc_swizzled(st, 16, L::QK_SBO, L::QK_SWIZZLE) + 2 * j, L::ID_SX, j > 0);
            // X = own2 ring2^T (K = dv), both K-major in 64-column blocks.
#pragma unroll
            for (int j = 0; j < DV / 16; ++j) {
                const uint32_t off = (j >> 2) * L::V_BLOCK + (j & 3) * 32;
                mma_bf16(tmem + L::COL_X, smem_desc_sw128(a2 + off, 16, 1024),
                         smem_desc_sw128(st + L::OFF_B2 + off, 16, 1024), L::ID_SX, j > 0);
            }
            mma_commit(&cx.bars[BB_SF]);
            mma_commit(&cx.bars[BB_EMPTY0 + s]);
            if (t == t1) mma_commit(&cx.bars[BB_OWNFREE]);   // the own tiles feed S / X only
            last = &cx.bars[BB_SF];
            lastp = step & 1;
        }
    }
    if (k_unit > 0) bwait(cx, BB_OWNFREE, (k_unit - 1) & 1);   // the last commit has landed
    bwd_drain(cx, last, lastp);
}

// Product issuer P (warp 1 + P, lane 0): P = 1 issues dV += A^T G (DKV) or
// dQ += dS K (DQ); P = 2 issues dK += dS^T Q (DKV). The operands formed by the
// row warps are read from TMEM, the ring's tiles as MN-major operands.
template <int DF, int DV, int MODE, int P>
__device__ __forceinline__ void bwd_issue_products(const BwdCtx& cx, uint32_t tmem) {
    using L = BwdLayout<DF, DV, MODE>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int own, bh, t0, t1;
        bwd_unit<MODE>(cx, u, own, bh, t0, t1);
        for (int t = t0; t <= t1; ++t, ++step) {
            const int s = step % L::STAGES;
            const int pb = step % L::NPB;
            bool ok = bwait(cx, BB_FULL0 + s, (step / L::STAGES) & 1) && bwait(cx, BB_PF0 + pb, (step / L::NPB) & 1);
            if (ok && t == t0 && k_unit >= 1) ok = bwait(cx, BB_ACCE, (k_unit - 1) & 1);
            if (!ok) { bwd_drain(cx, last, lastp); return; }
            tc_fence_after();
            const uint32_t st = cx.sbase + L::OFF_RING + s * L::STAGE_BYTES;
            const bool first = t == t0;
            if constexpr (MODE == MODE_DKV && P == 1) {
                // dV += A^T G: G of the ring, MN-major (rows = K = queries), 16 rows per K step.
#pragma unroll
                for (int j = 0; j < C / 16; ++j)
                    mma_bf16_ts(tmem + L::COL_ACC1, tmem + L::COL_P + 64 * pb + L::KSTEP_COLS * j,
                                smem_desc_sw128(st + L::OFF_B2 + j * 2048, L::V_BLOCK, 1024), L::ID_ACC1,
                                (!first || j > 0) ? 1u : 0u);
            } else {
                // dQ += dS K (DQ) or dK += dS^T Q (DKV): the ring's d'-wide tile, MN-major.
                const uint32_t a_ds = tmem + (MODE == MODE_DKV ? L::COL_D : L::COL_P + 64 * pb);
#pragma unroll
                for (int j = 0; j < C / 16; ++j)
                    mma_bf16_ts(tmem + L::COL_ACC2, a_ds + L::KSTEP_COLS * j,
                                smem_desc_swizzled(st + j * 16 * DF * 2, 16, L::QK_SBO, L::QK_SWIZZLE), L::ID_ACC2,
                                (!first || j > 0) ? 1u : 0u);
            }
            mma_commit(&cx.bars[BB_EMPTY0 + s]);
            mma_commit(&cx.bars[P == 1 ? BB_AFREE10 + pb : BB_AFREE2]);
            if (t == t1) mma_commit(&cx.bars[BB_ACCF]);
            last = &cx.bars[P == 1 ? BB_AFREE10 + pb : BB_AFREE2];
            lastp = (step / L::NPB) & 1;
        }
    }
    if (last != nullptr) bwait(cx, static_cast<int>(last - cx.bars), lastp);   // the last commit has landed
    bwd_drain(cx, last, lastp);
}

__device__ __forceinline__ void ld_shared_f2(uint32_t saddr, float& a, float& b) {
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(a), "=f"(b) : "r"(saddr) : "memory");
}

// ------------------------------------------------------------------ row warps (4..19)
// Thread = (row r of the unit's own tile = TMEM lane r, column group cg): each
// step it reads its 32 columns of S and X, forms the bf16 operands of those 32
// columns and, at the end of a unit, writes its share of the unit's results.
//
// DQ works on dy itself: with X' = dy V^T and c'_i = dy_i . y_i,
//     ds_ij = (X'_ij - c'_i)(1 + s_ij) / den_i,
// so the sweep over key tiles 0..qt accumulates den_i (the masked row sums of
// A) beside dQ' = sum_j (X'_ij - c'_i)(1 + s_ij) k_j, and the unit ends with
// dq_i = dQ'_i / den_i, g_i = dy_i / den_i (bf16, for DKV) and c_i = g_i . y_i.
template <int DF, int DV, int MODE>
__device__ __forceinline__ void bwd_rows(const BwdCtx& cx, uint32_t tmem, int wq, int cg, int lane,
                                         const __nv_bfloat16* __restrict__ y, const __nv_bfloat16* __restrict__ dy,
                                         __nv_bfloat16* __restrict__ G, float* __restrict__ cw,
                                         __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
                                         __nv_bfloat16* __restrict__ dv) {
    using L = BwdLayout<DF, DV, MODE>;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tl = tmem + lane_off;
    float* red = reinterpret_cast<float*>(cx.red);
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int own, bh, t0, t1;
        bwd_unit<MODE>(cx, u, own, bh, t0, t1);
        const int row = own * C + r;                         // this thread's row of the sequence
        const bool real = row < cx.N;
        const size_t vrow = ((size_t)bh * cx.N + (real ? row : 0)) * DV;   // row offset in y, dy, dv
        float l0 = 0.f, l1 = 0.f;                            // DQ: partial row sum of A
        float crow = 0.f;                                    // DQ: c'_i = dy_i . y_i
        if constexpr (MODE == MODE_DQ) {
            if (real) {
                const uint4* dyp = reinterpret_cast<const uint4*>(dy + vrow);
                const uint4* yp = reinterpret_cast<const uint4*>(y + vrow);
#pragma unroll 4
                for (int p = 0; p < DV / 8; ++p) {
                    const uint4 a = __ldg(dyp + p), b = __ldg(yp + p);
                    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        crow = fmaf(__uint_as_float(wa[e] << 16), __uint_as_float(wb[e] << 16), crow);
                        crow = fmaf(__uint_as_float(wa[e] & 0xFFFF0000u), __uint_as_float(wb[e] & 0xFFFF0000u), crow);
                    }
                }
            }
        }
        for (int t = t0; t <= t1; ++t, ++step) {
            if (!bwait(cx, BB_SF, step & 1)) return;
            tc_fence_after();
            float sv[32], xv[32];
            tmem_ld16(tl + L::COL_S + 32 * cg, sv);
            tmem_ld16(tl + L::COL_S + 32 * cg + 16, sv + 16);
            tmem_ld16(tl + L::COL_X + 32 * cg, xv);
            tmem_ld16(tl + L::COL_X + 32 * cg + 16, xv + 16);
            tmem_ld_wait();
            if constexpr (L::SEP) {
                tc_fence_before();
                mbar_arrive(&cx.bars[BB_SXFREE]);            // S / X may be overwritten
            }
            const bool diag = t == own;
            uint32_t cb = 0;
            if constexpr (MODE == MODE_DKV) {
                // c of the step's query tile, in the ring stage (its copy completed on FULL).
                const int s = step % L::STAGES;
                if (!bwait(cx, BB_FULL0 + s, (step / L::STAGES) & 1)) return;
                cb = cx.sbase + L::OFF_RING + s * L::STAGE_BYTES + L::OFF_CB;
            }
            uint32_t pa[16], pd[16];
            // One column pair: Taylor weight a (DKV: operand; DQ: row sum) and the
            // score gradient d, both zero where `keep` is false.
            auto pair = [&](int m, bool keep0, bool keep1) {
                float c0 = crow, c1 = crow;
                if constexpr (MODE == MODE_DKV) ld_shared_f2(cb + 4 * (32 * cg + 2 * m), c0, c1);
                float d0, d1, a0, a1;
                dscore_pair(xv[2 * m], xv[2 * m + 1], c0, c1, sv[2 * m], sv[2 * m + 1], d0, d1);
                taylor_pair(sv[2 * m], sv[2 * m + 1], a0, a1);
                if (!keep0) { d0 = 0.f; a0 = 0.f; }
                if (!keep1) { d1 = 0.f; a1 = 0.f; }
                pd[m] = pack_bf16x2(d0, d1);
                if constexpr (MODE == MODE_DKV) pa[m] = pack_bf16x2(a0, a1);
                else add_pair(l0, l1, a0, a1);
            };
            if (diag) {
                // Diagonal tile: DQ keeps key <= query (column <= row); DKV keeps
                // query >= key (column >= row).
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const int j0 = 32 * cg + 2 * m;
                    pair(m, MODE == MODE_DKV ? j0 >= r : j0 <= r, MODE == MODE_DKV ? j0 + 1 >= r : j0 + 1 <= r);
                }
            } else {
#pragma unroll
                for (int m = 0; m < 16; ++m) pair(m, true, true);
            }
            if constexpr (L::SEP) {
                // The previous step's products have read the operand region.
                // (DQ: the products of step - 2, which read this operand buffer.)
                if (step >= L::NPB && !bwait(cx, BB_AFREE10 + step % L::NPB, (step / L::NPB - 1) & 1)) return;
                if (L::NPI > 1 && step >= 1 && !bwait(cx, BB_AFREE2, (step - 1) & 1)) return;
                tc_fence_after();
            }
            // K steps 2cg and 2cg+1 of the products.
            const uint32_t k0c = L::KSTEP_COLS * (2 * cg), k1c = L::KSTEP_COLS * (2 * cg + 1);
            if constexpr (MODE == MODE_DKV) {
                tmem_st8(tl + L::COL_P + k0c, pa);
                tmem_st8(tl + L::COL_P + k1c, pa + 8);
                tmem_st8(tl + L::COL_D + k0c, pd);
                tmem_st8(tl + L::COL_D + k1c, pd + 8);
            } else {
                const uint32_t pcol = L::COL_P + 64 * (step % L::NPB);
                tmem_st8(tl + pcol + k0c, pd);
                tmem_st8(tl + pcol + k1c, pd + 8);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&cx.bars[BB_PF0 + step % L::NPB]);
        }
        // ---- the unit's results
        if constexpr (MODE == MODE_DQ) {
            // den_i = the groups' partial sums (exchanged through shared memory).
            float* lsum = red + (k_unit & 1) * kRowGroups * 128;
            float* csum = red + (2 + (k_unit & 1)) * kRowGroups * 128;
            lsum[cg * 128 + r] = l0 + l1;
            mbar_arrive(&cx.bars[BB_LSUM]);
            if (!bwait(cx, BB_LSUM, k_unit & 1)) return;
            float den = 0.f;
#pragma unroll
            for (int g2 = 0; g2 < kRowGroups; ++g2) den += lsum[g2 * 128 + r];
            const float inv = 1.0f / den;                    // den >= (row + 1) / 2
            // g = dy / den (bf16, the operand of DKV's products) and c = g . y over this
            // group's dv / groups columns; group 0 adds the partial c. Rows past the end
            // are 0. This needs den only, so it runs while the last products complete.
            constexpr int CPG = DV / kRowGroups;             // columns per group: 16 or 32
            uint4* gp = reinterpret_cast<uint4*>(G + ((size_t)bh * cx.Npad + row) * DV + cg * CPG);
            float c = 0.f;
            if (real) {
                const uint4* dyp = reinterpret_cast<const uint4*>(dy + vrow + cg * CPG);
                const uint4* yp = reinterpret_cast<const uint4*>(y + vrow + cg * CPG);
#pragma unroll
                for (int p = 0; p < CPG / 8; ++p) {
                    const uint4 a = __ldg(dyp + p), b = __ldg(yp + p);
                    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
                    float gf[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        gf[2 * e] = __uint_as_float(wa[e] << 16) * inv;
                        gf[2 * e + 1] = __uint_as_float(wa[e] & 0xFFFF0000u) * inv;
                    }
                    // c from the rounded g that DKV's products use, so that the column
                    // sums over j of a_ij (g_i . v_j - c_i) stay consistent.
                    const uint4 gr = pack_bf16x8(gf);
                    const uint32_t wg[4] = {gr.x, gr.y, gr.z, gr.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        c = fmaf(__uint_as_float(wg[e] << 16), __uint_as_float(wb[e] << 16), c);
                        c = fmaf(__uint_as_float(wg[e] & 0xFFFF0000u), __uint_as_float(wb[e] & 0xFFFF0000u), c);
                    }
                    gp[p] = gr;
                }
            } else {
#pragma unroll
                for (int p = 0; p < CPG / 8; ++p) gp[p] = make_uint4(0, 0, 0, 0);
            }
            csum[cg * 128 + r] = c;
            mbar_arrive(&cx.bars[BB_CSUM]);
            // dq_i = dQ'_i / den_i: 16-column slices of the accumulator by group.
            if (!bwait(cx, BB_ACCF, k_unit & 1)) return;
            tc_fence_after();
#pragma unroll
            for (int i = cg; i < DF / 16; i += kRowGroups) {
                float acc[16];
                tmem_ld16(tl + L::COL_ACC2 + 16 * i, acc);
                tmem_ld_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] *= inv;
                if (real) {
                    uint4* op = reinterpret_cast<uint4*>(dq + ((size_t)bh * cx.N + row) * DF + 16 * i);
                    op[0] = pack_bf16x8(acc);
                    op[1] = pack_bf16x8(acc + 8);
                }
            }
            tc_fence_before();
            mbar_arrive(&cx.bars[BB_ACCE]);                  // the accumulator may be reused
            if (cg == 0) {
                if (!bwait(cx, BB_CSUM, k_unit & 1)) return;
                float ct = 0.f;
#pragma unroll
                for (int g2 = 0; g2 < kRowGroups; ++g2) ct += csum[g2 * 128 + r];
                cw[(size_t)bh * cx.Npad + row] = ct;
            }
        } else {
            // Accumulator read-out: 16-column slice i (dK slices first, then dV) by
            // group i mod groups.
            if (!bwait(cx, BB_ACCF, k_unit & 1)) return;
            tc_fence_after();
            constexpr int NS2 = DF / 16, NS = NS2 + DV / 16;
#pragma unroll
            for (int i = cg; i < NS; i += kRowGroups) {
                float a[16];
                const bool second = i < NS2;
                tmem_ld16(tl + (second ? L::COL_ACC2 + 16 * i : L::COL_ACC1 + 16 * (i - NS2)), a);
                tmem_ld_wait();
                if (real) {
                    uint4* op = second ? reinterpret_cast<uint4*>(dk + ((size_t)bh * cx.N + row) * DF + 16 * i)
                                       : reinterpret_cast<uint4*>(dv + vrow + 16 * (i - NS2));
                    op[0] = pack_bf16x8(a);
                    op[1] = pack_bf16x8(a + 8);
                }
            }
            tc_fence_before();
            mbar_arrive(&cx.bars[BB_ACCE]);                  // the accumulators may be reused
        }
    }
}

template <int DF, int DV, int MODE>
__global__ void __launch_bounds__(kBwdThreads, 1)
la_bwd_kernel(const __grid_constant__ CUtensorMap m_own1, const __grid_constant__ CUtensorMap m_own2,
              const __grid_constant__ CUtensorMap m_ring1, const __grid_constant__ CUtensorMap m_ring2,
              const __nv_bfloat16* __restrict__ y, const __nv_bfloat16* __restrict__ dy,
              __nv_bfloat16* __restrict__ G, float* __restrict__ cw, __nv_bfloat16* __restrict__ dq,
              __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv, int N, int Npad, int BH, int nt,
              unsigned* status, unsigned debug) {
    using L = BwdLayout<DF, DV, MODE>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + 8 * BB_NUM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BAR + 8 * BB_NUM + 4);
    const BwdCtx cx{sbase, bars, smem + L::OFF_RED, abort_flag, status, N, Npad, BH, nt, nt * BH};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int b = 0; b < BB_NUM; ++b) {
            uint32_t count = 1;
            if (b == BB_SXFREE || b == BB_PF0 || b == BB_PF0 + 1 || b == BB_ACCE || b == BB_LSUM || b == BB_CSUM)
                count = kRowThreads;
            if (b >= BB_EMPTY0 && b < BB_EMPTY0 + L::STAGES) count = 1 + L::NPI;
            if (b == BB_ACCF) count = L::NPI;
            mbar_init(&bars[b], count);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, L::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dependency_wait();                                  // inputs and workspace may come from earlier kernels
    const bool skip_mma = (debug & DEBUG_SKIP_MMA) != 0;    // testing: issue nothing, every waiter times out

    if (warp == 0) {
        if (lane == 0) bwd_producer<DF, DV, MODE>(cx, BwdMaps{&m_own1, &m_own2, &m_ring1, &m_ring2}, cw);
    } else if (warp == 1) {
        if (lane == 0 && !skip_mma) bwd_issue_sx<DF, DV, MODE>(cx, tmem);
    } else if (warp == 2) {
        if (lane == 0 && !skip_mma) bwd_issue_products<DF, DV, MODE, 1>(cx, tmem);
    } else if (warp == 3) {
        if constexpr (L::NPI >= 2)
            if (lane == 0 && !skip_mma) bwd_issue_products<DF, DV, MODE, 2>(cx, tmem);
    } else {
        bwd_rows<DF, DV, MODE>(cx, tmem, warp & 3, (warp - 4) >> 2, lane, y, dy, G, cw, dq, dk, dv);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

template <int DF, int DV, int MODE>
cudaError_t launch_mode(const LaBackwardArgs& a, const CUtensorMap& own1, const CUtensorMap& own2,
                        const CUtensorMap& ring1, const CUtensorMap& ring2, __nv_bfloat16* G, float* cw, int Npad,
                        int num_sms, cudaStream_t stream) {
    using L = BwdLayout<DF, DV, MODE>;
    using bf = __nv_bfloat16;
    const int BH = a.B * a.H, nt = Npad / C;
    auto kern = la_bwd_kernel<DF, DV, MODE>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<long long>((long long)nt * BH, num_sms);
    return launch_pdl(kern, dim3(grid), dim3(kBwdThreads), L::SMEM_BYTES, stream, own1, own2, ring1, ring2,
                      static_cast<const bf*>(a.y), static_cast<const bf*>(a.dy), G, cw, static_cast<bf*>(a.dq),
                      static_cast<bf*>(a.dk), static_cast<bf*>(a.dv), a.N, Npad, BH, nt, a.status, a.debug);
}

template <int DF, int DV>
cudaError_t launch_typed(const LaBackwardArgs& a, int num_sms, cudaStream_t stream) {
    const int BH = a.B * a.H;
    const int Npad = (a.N + C - 1) / C * C;
    auto* G = static_cast<__nv_bfloat16*>(a.workspace);
    auto* cw = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) + la_backward_g_bytes(a));
    CUtensorMap mq, mk, mv, mdy, mg;
    if (!make_tmap_bf16_3d_swizzle(&mq, a.q, DF, a.N, BH, DF, C, DF * 2) ||
        !make_tmap_bf16_3d_swizzle(&mk, a.k, DF, a.N, BH, DF, C, DF * 2) ||
        !make_tmap_bf16_3d_swizzle(&mv, a.v, DV, a.N, BH, 64, C, 128) ||
        !make_tmap_bf16_3d_swizzle(&mdy, a.dy, DV, a.N, BH, 64, C, 128) ||
        !make_tmap_bf16_3d_swizzle(&mg, G, DV, Npad, BH, 64, C, 128))
        return cudaErrorInvalidValue;
    cudaError_t e = launch_mode<DF, DV, MODE_DQ>(a, mq, mdy, mk, mv, G, cw, Npad, num_sms, stream);
    if (e != cudaSuccess) return e;
    return launch_mode<DF, DV, MODE_DKV>(a, mk, mv, mq, mg, G, cw, Npad, num_sms, stream);
}

}  // namespace

size_t la_backward_g_bytes(const LaBackwardArgs& a) {
    const size_t Npad = (size_t)(a.N + C - 1) / C * C;
    return (size_t)a.B * a.H * Npad * a.d_v * 2;
}

size_t la_backward_workspace(int B, int H, int N, int d_feat, int d_v) {
    const size_t Npad = (size_t)(N + C - 1) / C * C;
    (void)d_feat;
    return (size_t)B * H * Npad * (d_v * 2 + 4);
}

bool la_backward_supported(int d_feat, int d_v) {
    return (d_feat == 16 || d_feat == 32) && (d_v == 64 || d_v == 128);
}

cudaError_t launch_la_backward(const LaBackwardArgs& a, int num_sms, cudaStream_t stream) {
    if (!la_backward_supported(a.d_feat, a.d_v)) return cudaErrorInvalidValue;
    if (a.d_feat == 16 && a.d_v == 64) return launch_typed<16, 64>(a, num_sms, stream);
    if (a.d_feat == 16 && a.d_v == 128) return launch_typed<16, 128>(a, num_sms, stream);
    if (a.d_feat == 32 && a.d_v == 64) return launch_typed<32, 64>(a, num_sms, stream);
    return launch_typed<32, 128>(a, num_sms, stream);
}

}  // namespace based

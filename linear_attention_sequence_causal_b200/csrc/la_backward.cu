// Backward (training) pass of causal Taylor linear attention on the tensor cores.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED) §5 "Execution stages" names prefill during training; the
// forward is y_i = sum_{j<=i} a_ij v_j / den_i, a_ij = 1 + s_ij + s_ij^2/2,
// s_ij = q_i.k_j, den_i = sum_{j<=i} a_ij. For an upstream gradient dy:
//     g_i   = dy_i / den_i,   c_i = g_i . y_i,
//     ds_ij = (g_i . v_j - c_i) (1 + s_ij)         (j <= i, else 0),
//     dq_i  = sum_j ds_ij k_j,   dk_j = sum_i ds_ij q_i,   dv_j = sum_i a_ij g_i.
// Three persistent kernels, each one CTA per SM walking 128-row units longest
// first and sweeping the 128-row tiles of the other side:
//   DEN  unit = query tile: S = Q K^T (M=128 N=128 K=d') -> den = row sums of
//        the masked A; then G = dy / den (bf16) and c = g . y to the workspace
//        (rows padded to a multiple of 128 with zeros);
//   DQ   unit = query tile: S = Q K^T, X = G V^T (K=dv); dS = (X - c)(1 + S),
//        bf16 in TMEM; dQ += dS K (A operand in TMEM, K as an MN-major operand);
//   DKV  unit = key tile: S^T = K Q^T, X^T = V G^T; A^T and dS^T in TMEM;
//        dV += A^T G and dK += dS^T Q (G and Q as MN-major operands).
// Each d'-wide tile (Q, K) sits in shared memory under the swizzle of its row
// width and serves both as a K-major operand (rows = M or N) and, read along
// its rows, as an MN-major operand (rows = K); each dv-wide tile (V, G) sits in
// 64-column blocks under the 128-byte swizzle and serves both ways likewise.
// Roles (192 threads): warp 0 lane 0 loads by TMA (the unit's own tile(s) and a
// 2-stage ring of the other side's tiles); warp 1 allocates TMEM and lane 0
// issues every MMA; warps 2-5 (thread = row = TMEM lane) form A / dS and write
// the unit's results. Every hand-off is an mbarrier; every wait is bounded.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma_host.h"

namespace based {
namespace {

using namespace tc;

constexpr int C = 128;
constexpr int kBwdThreads = 192;
enum { MODE_DEN = 0, MODE_DQ = 1, MODE_DKV = 2 };

template <int DF, int DV, int MODE>
struct BwdLayout {
    static constexpr int QK_SWIZZLE = DF * 2;
    static constexpr uint32_t QK_BYTES = C * DF * 2;          // d'-wide tile: 128 rows of d' bf16
    static constexpr uint32_t QK_SBO = 8 * DF * 2;            // 8 rows
    static constexpr uint32_t V_BLOCK = C * 128;              // 64 columns x 128 rows, 128-byte swizzle
    static constexpr uint32_t V_BYTES = C * DV * 2;           // dv-wide tile
    static constexpr bool WIDE = MODE != MODE_DEN;            // a dv-wide tile on each side
    static constexpr bool HAS_C = MODE == MODE_DKV;           // c of the stage's query tile
    static constexpr uint32_t STAGE_BYTES = QK_BYTES + (WIDE ? V_BYTES : 0) + (HAS_C ? 1024 : 0);
    static constexpr uint32_t OFF_A1 = 0;                     // own d'-wide tile
    static constexpr uint32_t OFF_A2 = OFF_A1 + QK_BYTES;     // own dv-wide tile
    static constexpr uint32_t OFF_RING = OFF_A2 + (WIDE ? V_BYTES : 0);
    static constexpr uint32_t OFF_B2 = QK_BYTES;              // within a stage
    static constexpr uint32_t OFF_CB = QK_BYTES + (WIDE ? V_BYTES : 0);
    static constexpr uint32_t OFF_BAR = OFF_RING + 2 * STAGE_BYTES;
    static constexpr uint32_t SMEM_NEED = OFF_BAR + 256 + 1024;    // + alignment slack
    // At least 116 KB, so that one CTA sits on an SM and owns all 512 TMEM columns.
    static constexpr uint32_t SMEM_BYTES = SMEM_NEED > 116 * 1024 ? SMEM_NEED : 116 * 1024;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(QK_BYTES % 1024 == 0 && V_BYTES % 1024 == 0 && STAGE_BYTES % 1024 == 0, "tile alignment");
    // TMEM: S [0,128), X [128,256) (dS^T overlays X in DKV), then dV (DKV) and dQ / dK.
    static constexpr uint32_t COL_S = 0, COL_X = 128, COL_ACC1 = 256;
    static constexpr uint32_t COL_ACC2 = MODE == MODE_DKV ? 256 + DV : 256;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_ACC2 + DF <= TMEM_COLS, "tensor memory");
    static constexpr uint32_t ID_SX = idesc_bf16_f32(128, C, false, false);      // S, X: both operands K-major
    static constexpr uint32_t ID_ACC1 = idesc_bf16_f32(128, DV, false, true);    // dV += A^T G
    static constexpr uint32_t ID_ACC2 = idesc_bf16_f32(128, DF, false, true);    // dQ += dS K, dK += dS^T Q
};

enum {
    BB_FULL0, BB_FULL1,       // TMA: ring stage s landed
    BB_EMPTY0, BB_EMPTY1,     // MMA commit: ring stage s read
    BB_OWNFULL,               // TMA: the unit's own tile(s) landed
    BB_OWNFREE,               // MMA commit: the unit's own tiles no longer read
    BB_SF,                    // MMA commit: S (and X) of the step ready
    BB_PF,                    // row warps: A / dS of the step written (DQ, DKV)
    BB_SFREE,                 // S / X columns free again (DEN: row warps read S; else MMA commit)
    BB_ACCF,                  // MMA commit: the unit's accumulators complete
    BB_ACCE,                  // row warps: accumulators read out
    BB_NUM
};

struct BwdCtx {
    uint32_t sbase;
    uint64_t* bars;
    volatile int* abort_flag;
    unsigned* status;
    int N, Npad, BH, nt, nunits;
};

__device__ __forceinline__ bool bwait(const BwdCtx& cx, int bar, uint32_t parity) {
    return mbar_wait(&cx.bars[bar], parity, cx.abort_flag, cx.status);
}

// Unit u: its own tile index, its head and its sweep of the other side's tiles
// [t0, t1]. DEN and DQ: query tile qt (longest first) against key tiles 0..qt;
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
    const CUtensorMap* own1;   // d'-wide own tile (q for DEN/DQ, k for DKV)
    const CUtensorMap* own2;   // dv-wide own tile (G for DQ, v for DKV)
    const CUtensorMap* ring1;  // d'-wide ring tile (k for DEN/DQ, q for DKV)
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
        mbar_expect_tx(of, L::QK_BYTES + (L::WIDE ? L::V_BYTES : 0));
        tma_load_3d(cx.sbase + L::OFF_A1, m.own1, of, 0, own * C, bh);
        if constexpr (L::WIDE) {
#pragma unroll
            for (int h = 0; h < DV / 64; ++h)
                tma_load_3d(cx.sbase + L::OFF_A2 + h * L::V_BLOCK, m.own2, of, 64 * h, own * C, bh);
        }
        last = of;
        lastp = k_unit & 1;
        for (int t = t0; t <= t1; ++t, ++step) {
            const int s = step & 1;
            if (step >= 2 && !bwait(cx, BB_EMPTY0 + s, ((step >> 1) - 1) & 1)) { bwd_drain(cx, last, lastp); return; }
            uint64_t* full = &cx.bars[BB_FULL0 + s];
            const uint32_t st = cx.sbase + L::OFF_RING + s * L::STAGE_BYTES;
            mbar_expect_tx(full, L::QK_BYTES + (L::WIDE ? L::V_BYTES : 0) + (L::HAS_C ? C * 4 : 0));
            tma_load_3d(st, m.ring1, full, 0, t * C, bh);
            if constexpr (L::WIDE) {
#pragma unroll
                for (int h = 0; h < DV / 64; ++h)
                    tma_load_3d(st + L::OFF_B2 + h * L::V_BLOCK, m.ring2, full, 64 * h, t * C, bh);
            }
            if constexpr (L::HAS_C) bulk_load(st + L::OFF_CB, cw + (size_t)bh * cx.Npad + t * C, C * 4, full);
            last = full;
            lastp = (step >> 1) & 1;
        }
    }
    bwd_drain(cx, last, lastp);
}

// ------------------------------------------------------------------ MMA issuer (warp 1, lane 0)
template <int DF, int DV, int MODE>
__device__ __forceinline__ void bwd_issuer(const BwdCtx& cx, uint32_t tmem) {
    using L = BwdLayout<DF, DV, MODE>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    const uint32_t a1 = cx.sbase + L::OFF_A1, a2 = cx.sbase + L::OFF_A2;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int own, bh, t0, t1;
        bwd_unit<MODE>(cx, u, own, bh, t0, t1);
        for (int t = t0; t <= t1; ++t, ++step) {
            const int s = step & 1;
            const bool first = t == t0, lastt = t == t1;
            const uint32_t st = cx.sbase + L::OFF_RING + s * L::STAGE_BYTES;
            if (!bwait(cx, BB_FULL0 + s, (step >> 1) & 1)) { bwd_drain(cx, last, lastp); return; }
            if (first && !bwait(cx, BB_OWNFULL, k_unit & 1)) { bwd_drain(cx, last, lastp); return; }
            if (step >= 1 && !bwait(cx, BB_SFREE, (step - 1) & 1)) { bwd_drain(cx, last, lastp); return; }
            tc_fence_after();
            // S = own1 ring1^T (K = d'), both K-major.
#pragma unroll
            for (int j = 0; j < DF / 16; ++j)
                mma_bf16(tmem + L::COL_S, smem_desc_swizzled(a1, 16, L::QK_SBO, L::QK_SWIZZLE) + 2 * j,
                         smem_desc_swizzled(st, 16, L::QK_SBO, L::QK_SWIZZLE) + 2 * j, L::ID_SX, j > 0);
            if constexpr (L::WIDE) {
                // X = own2 ring2^T (K = dv), both K-major in 64-column blocks.
#pragma unroll
                for (int j = 0; j < DV / 16; ++j) {
                    const uint32_t off = (j >> 2) * L::V_BLOCK + (j & 3) * 32;
                    mma_bf16(tmem + L::COL_X, smem_desc_sw128(a2 + off, 16, 1024),
                             smem_desc_sw128(st + L::OFF_B2 + off, 16, 1024), L::ID_SX, j > 0);
                }
            }
            mma_commit(&cx.bars[BB_SF]);
            last = &cx.bars[BB_SF];
            lastp = step & 1;
            if constexpr (MODE == MODE_DEN) {
                mma_commit(&cx.bars[BB_EMPTY0 + s]);
                if (lastt) mma_commit(&cx.bars[BB_OWNFREE]);
                continue;
            }
            if (!bwait(cx, BB_PF, step & 1)) { bwd_drain(cx, last, lastp); return; }
            if (first && k_unit >= 1 && !bwait(cx, BB_ACCE, (k_unit - 1) & 1)) { bwd_drain(cx, last, lastp); return; }
            tc_fence_after();
            if constexpr (MODE == MODE_DKV) {
                // dV += A^T G: A^T (bf16, TMEM over S), G of the ring as MN-major (rows = K).
#pragma unroll
                for (int j = 0; j < C / 16; ++j)
                    mma_bf16_ts(tmem + L::COL_ACC1, tmem + L::COL_S + 8 * j,
                                smem_desc_sw128(st + L::OFF_B2 + j * 2048, L::V_BLOCK, 1024), L::ID_ACC1,
                                (!first || j > 0) ? 1u : 0u);
            }
            // dQ += dS K (DQ) or dK += dS^T Q (DKV): dS in TMEM (over S for DQ, over X for
            // DKV), the ring's d'-wide tile as MN-major, 16 rows per K step.
            const uint32_t a_ds = tmem + (MODE == MODE_DKV ? L::COL_X : L::COL_S);
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16_ts(tmem + L::COL_ACC2, a_ds + 8 * j,
                            smem_desc_swizzled(st + j * 16 * DF * 2, 16, L::QK_SBO, L::QK_SWIZZLE), L::ID_ACC2,
                            (!first || j > 0) ? 1u : 0u);
            mma_commit(&cx.bars[BB_EMPTY0 + s]);
            mma_commit(&cx.bars[BB_SFREE]);
            last = &cx.bars[BB_SFREE];
            lastp = step & 1;
            if (lastt) {
                mma_commit(&cx.bars[BB_ACCF]);
                mma_commit(&cx.bars[BB_OWNFREE]);
            }
        }
    }
    // The last commit has landed before the CTA (and its barriers) goes away.
    if (k_unit > 0 && !*cx.abort_flag) bwait(cx, BB_OWNFREE, (k_unit - 1) & 1);
    bwd_drain(cx, last, lastp);
}

__device__ __forceinline__ void ld_shared_f2(uint32_t saddr, float& a, float& b) {
    asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(a), "=f"(b) : "r"(saddr) : "memory");
}

// ------------------------------------------------------------------ row warps (2-5)
// Thread = row r of the unit's own tile = TMEM lane r (wq = lane quadrant).
template <int DF, int DV, int MODE>
__device__ __forceinline__ void bwd_rows(const BwdCtx& cx, uint32_t tmem, int wq, int lane,
                                         const __nv_bfloat16* __restrict__ y, const __nv_bfloat16* __restrict__ dy,
                                         __nv_bfloat16* __restrict__ G, float* __restrict__ cw,
                                         __nv_bfloat16* __restrict__ dq, __nv_bfloat16* __restrict__ dk,
                                         __nv_bfloat16* __restrict__ dv) {
    using L = BwdLayout<DF, DV, MODE>;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t ts = tmem + lane_off + L::COL_S, tx = tmem + lane_off + L::COL_X;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int own, bh, t0, t1;
        bwd_unit<MODE>(cx, u, own, bh, t0, t1);
        const int row = own * C + r;                         // this thread's row of the sequence
        float l0 = 0.f, l1 = 0.f;                            // DEN: row sum of A
        float crow = 0.f;                                    // DQ: c of this query row
        if constexpr (MODE == MODE_DQ) crow = cw[(size_t)bh * cx.Npad + row];
        for (int t = t0; t <= t1; ++t, ++step) {
            if (!bwait(cx, BB_SF, step & 1)) return;
            tc_fence_after();
            const bool diag = t == own;
            uint32_t cb = 0;
            if constexpr (MODE == MODE_DKV) {
                // c of the step's query tile, in the ring stage (its TMA completed on FULL).
                const int s = step & 1;
                if (!bwait(cx, BB_FULL0 + s, (step >> 1) & 1)) return;
                cb = cx.sbase + L::OFF_RING + s * L::STAGE_BYTES + L::OFF_CB;
            }
#pragma unroll 1
            for (int c2 = 0; c2 < C / 16; ++c2) {
                float sv[16], xv[16];
                tmem_ld16(ts + 16 * c2, sv);
                if constexpr (L::WIDE) tmem_ld16(tx + 16 * c2, xv);
                tmem_ld_wait();
                uint32_t pa[8], pd[8];
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const int j0 = 16 * c2 + 2 * m;            // column of the pair's low half
                    // Causal mask on the diagonal tile: DEN / DQ keep key <= query
                    // (column <= row); DKV keeps query >= key (column >= row).
                    const bool k0 = !diag || (MODE == MODE_DKV ? j0 >= r : j0 <= r);
                    const bool k1 = !diag || (MODE == MODE_DKV ? j0 + 1 >= r : j0 + 1 <= r);
                    float a0, a1;
                    taylor_pair(sv[2 * m], sv[2 * m + 1], a0, a1);
                    a0 = k0 ? a0 : 0.f;
                    a1 = k1 ? a1 : 0.f;
                    if constexpr (MODE == MODE_DEN) {
                        add_pair(l0, l1, a0, a1);
                    } else {
                        float c0 = crow, c1 = crow;
                        if constexpr (MODE == MODE_DKV) ld_shared_f2(cb + 4 * j0, c0, c1);
                        const float d0 = k0 ? (xv[2 * m] - c0) * (1.f + sv[2 * m]) : 0.f;
                        const float d1 = k1 ? (xv[2 * m + 1] - c1) * (1.f + sv[2 * m + 1]) : 0.f;
                        pd[m] = pack_bf16x2(d0, d1);
                        pa[m] = pack_bf16x2(a0, a1);
                    }
                }
                if constexpr (MODE == MODE_DQ) tmem_st8(ts + 8 * c2, pd);                 // dS over S
                if constexpr (MODE == MODE_DKV) {
                    tmem_st8(ts + 8 * c2, pa);                                              // A^T over S
                    tmem_st8(tx + 8 * c2, pd);                                              // dS^T over X
                }
            }
            if constexpr (MODE == MODE_DEN) {
                tc_fence_before();
                mbar_arrive(&cx.bars[BB_SFREE]);             // S read: the next step may overwrite it
            } else {
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(&cx.bars[BB_PF]);
            }
        }
        // ---- the unit's results for this row
        if constexpr (MODE == MODE_DEN) {
            // g = dy / den (bf16, the operand of the later products) and c = g . y;
            // rows past the sequence end are zero.
            const float den = l0 + l1;
            uint4* gp = reinterpret_cast<uint4*>(G + ((size_t)bh * cx.Npad + row) * DV);
            float c = 0.f;
            if (row < cx.N) {
                const uint4* dyp = reinterpret_cast<const uint4*>(dy + ((size_t)bh * cx.N + row) * DV);
                const uint4* yp = reinterpret_cast<const uint4*>(y + ((size_t)bh * cx.N + row) * DV);
                const float inv = 1.0f / den;                // den >= (row + 1) / 2
#pragma unroll 1
                for (int p = 0; p < DV / 8; ++p) {
                    const uint4 a = __ldg(dyp + p), b = __ldg(yp + p);
                    const uint32_t wa[4] = {a.x, a.y, a.z, a.w}, wb[4] = {b.x, b.y, b.z, b.w};
                    float gf[8];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        gf[2 * e] = __uint_as_float(wa[e] << 16) * inv;
                        gf[2 * e + 1] = __uint_as_float(wa[e] & 0xFFFF0000u) * inv;
                    }
                    // c from the rounded g that the products use, so that the row's
                    // sum over j of a_ij (g . v_j - c_i) stays zero up to accumulation order.
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
#pragma unroll 1
                for (int p = 0; p < DV / 8; ++p) gp[p] = make_uint4(0, 0, 0, 0);
            }
            cw[(size_t)bh * cx.Npad + row] = c;
        } else {
            if (!bwait(cx, BB_ACCF, k_unit & 1)) return;
            tc_fence_after();
            const uint32_t t2 = tmem + lane_off + L::COL_ACC2;
            float a2[DF];
#pragma unroll
            for (int h = 0; h < DF / 16; ++h) tmem_ld16(t2 + 16 * h, a2 + 16 * h);
            tmem_ld_wait();
            __nv_bfloat16* out2 = MODE == MODE_DKV ? dk : dq;
            if (row < cx.N) {
                uint4* op = reinterpret_cast<uint4*>(out2 + ((size_t)bh * cx.N + row) * DF);
#pragma unroll
                for (int p = 0; p < DF / 8; ++p) op[p] = pack_bf16x8(a2 + 8 * p);
            }
            if constexpr (MODE == MODE_DKV) {
                const uint32_t t1a = tmem + lane_off + L::COL_ACC1;
                uint4* op = reinterpret_cast<uint4*>(dv + ((size_t)bh * cx.N + (row < cx.N ? row : 0)) * DV);
#pragma unroll 1
                for (int h = 0; h < DV / 16; ++h) {
                    float a1[16];
                    tmem_ld16(t1a + 16 * h, a1);
                    tmem_ld_wait();
                    if (row < cx.N) {
                        op[2 * h] = pack_bf16x8(a1);
                        op[2 * h + 1] = pack_bf16x8(a1 + 8);
                    }
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
    const BwdCtx cx{sbase, bars, abort_flag, status, N, Npad, BH, nt, nt * BH};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int b = 0; b < BB_NUM; ++b) {
            uint32_t count = 1;
            if (b == BB_PF || b == BB_ACCE || (b == BB_SFREE && MODE == MODE_DEN)) count = 128;
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
        if (lane == 0 && !skip_mma) bwd_issuer<DF, DV, MODE>(cx, tmem);
    } else {
        bwd_rows<DF, DV, MODE>(cx, tmem, warp & 3, lane, y, dy, G, cw, dq, dk, dv);
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
    CUtensorMap mq, mk, mv, mg;
    if (!make_tmap_bf16_3d_swizzle(&mq, a.q, DF, a.N, BH, DF, C, DF * 2) ||
        !make_tmap_bf16_3d_swizzle(&mk, a.k, DF, a.N, BH, DF, C, DF * 2) ||
        !make_tmap_bf16_3d_swizzle(&mv, a.v, DV, a.N, BH, 64, C, 128) ||
        !make_tmap_bf16_3d_swizzle(&mg, G, DV, Npad, BH, 64, C, 128))
        return cudaErrorInvalidValue;
    cudaError_t e = launch_mode<DF, DV, MODE_DEN>(a, mq, mq, mk, mk, G, cw, Npad, num_sms, stream);
    if (e != cudaSuccess) return e;
    e = launch_mode<DF, DV, MODE_DQ>(a, mq, mg, mk, mv, G, cw, Npad, num_sms, stream);
    if (e != cudaSuccess) return e;
    return launch_mode<DF, DV, MODE_DKV>(a, mk, mv, mq, mg, G, cw, Npad, num_sms, stream);
}

}  // namespace

size_t la_backward_g_bytes(const LaBackwardArgs& a) {
    const size_t Npad = (size_t)(a.N + C - 1) / C * C;
    return (size_t)a.B * a.H * Npad * a.d_v * 2;
}

size_t la_backward_workspace(int B, int H, int N, int d_v) {
    const size_t Npad = (size_t)(N + C - 1) / C * C;
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

// Tensor-core chunked prefill of causal Taylor linear attention for the shapes
// whose state does not fit one SM's tensor memory (d' = 32, or dv = 128):
// y_i = sum_{j<=i} a_ij v_j / sum_{j<=i} a_ij, a_ij = 1 + s + s^2/2, s = q_i.k_j.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), App. B "Forward / Generation Prefill" computes each tile as
// a quadratic on-diagonal part under a local causal mask plus a linear
// off-diagonal part read from the cumulative state of the earlier chunks. At
// d' = 32 and dv = 128 the folded state [S | z] is 561 x 129 fp32 (290 KB), more
// than the 256 KB of tensor memory of one SM, so the state and the outputs are
// computed by two kernels ("Gated Slot Attention", App. A.1: the chunkwise form
// is recurrent across chunks and parallel within one):
//
// la_prefix_kernel (one CTA per head and 128-feature tile, two per SM) sweeps
// the tokens once: [S | z] += phi(K)^T [V | 1] per 64-token step, S by the
// tensor cores (M=128 features, N=dv, K=64, fp32 in TMEM), z in fp32 on the
// CUDA cores. At every chunk boundary (every L tokens) it writes the state of
// the tokens before it -- the state a chunk starts from -- to the workspace:
// S rounded to bf16, z in fp32. At the end it writes the final S and z.
//
// la_quad_kernel (persistent, one CTA per SM) computes y. A unit is (query tile
// qt of 128 tokens, head bh) in chunk ch = qt / (L/128); it runs "steps", each an
// M=128 K=128 product into the O accumulator:
//   virtual steps (ch > 0), one per 128-feature tile f of the folded features:
//     P  = phi(Q_qt)[:, f] in bf16 (formed from q by the A warps, no MMA),
//     O += P S_ch[f, :]               N=dv  (the chunk-start state, by TMA)
//     l += phi(Q_qt)[:, f] . z_ch[f]  (fp32, the denominator's state part)
//   intra steps, key tiles kt of the chunk up to qt:
//     S  = Q_qt K_kt^T                M=128 N=128 K=d'   -> TMEM
//     P  = 1 + S + S^2/2 (causal mask on the diagonal tile), bf16 over S in TMEM;
//     l += row sums of P (fp32, before rounding)
//     O += P V_kt                     N=dv  (P in TMEM)
//   y = O / l.
// With a chunk at least as long as the sequence there are no virtual steps and
// this is the quadratic form (every key tile at or below the diagonal), which
// the coarse-decay path uses.
//
// Roles of la_quad_kernel (512 threads):
//   warp 0      lane 0: TMA loads into a 4-stage ring: the unit's Q tile, and
//               per step either K and V tiles, or (virtual step) a copy of the
//               Q tile, the state tile and its z slice (rows past the
//               sequence or the state read as 0);
//   warp 1      allocates TMEM; lane 0 issues S of every intra step into S
//               buffer (step mod 3) and releases the buffer for virtual steps;
//   warps 2, 3  lane 0: O_g += P V of the steps of parity g, into accumulator
//               O_g (two issuers keep the tensor pipe busy: one thread alone
//               issues an MMA about every 117 cycles, while an M=128 N=128
//               K=16 product takes 64); one at dv = 128, where TMEM holds one O;
//   warps 4-15  three groups of four warps: group g forms P of the steps with
//               step mod 3 == g (thread = query row = TMEM lane), and at the end
//               of a unit writes y = (O_0 + O_1) / l for its column blocks.
// Every hand-off is an mbarrier; every wait is bounded.
#include <algorithm>
#include <utility>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma_host.h"

namespace based {
namespace {

using namespace tc;

constexpr int C = 128;               // query and key tile
constexpr int kStages = 4;
constexpr int kBufs = 3;            // S / P buffers in TMEM
constexpr int kQuadThreads = 512;
constexpr int kZSlice = 128 * 4;    // bytes of one 128-feature z slice

// Folded feature f of [1, x_a, x_a x_b (a <= b, a-major)] as x[a] * x[b] * coef,
// x[DF] standing for the constant; coef 0 past the last feature. The order of
// the state rows in the workspace, and of phi(q) in the virtual steps.
struct FeatPair {
    int a, b;
    float coef;
};
__host__ __device__ constexpr FeatPair feat_pair(int DF, int f) {
    if (f == 0) return FeatPair{DF, DF, 1.0f};
    if (f <= DF) return FeatPair{f - 1, DF, 1.0f};
    int p = f - 1 - DF, a = 0;
    while (a < DF && p >= DF - a) { p -= DF - a; ++a; }
    if (a >= DF) return FeatPair{DF, DF, 0.0f};
    return FeatPair{a, a + p, p == 0 ? kSqrtHalf : 1.0f};
}

// Tiles of 128 folded features (2 at d' = 16, 5 at d' = 32).
__host__ __device__ constexpr int feature_tiles(int DF) { return (sym_feature_dim(DF) + 127) / 128; }

template <int DF, int DV>
struct QuadLayout {
    // Q and K tiles: K-major rows of d' bf16 (32 or 64 bytes) under the swizzle
    // of that width, 8-row atoms. V tile: MN-major under the 128-byte swizzle,
    // one 128-key x 64-value block per 64 values (a state tile has the same
    // layout with features in place of keys).
    static constexpr int QK_SWIZZLE = DF * 2;
    static constexpr uint32_t QK_BYTES = C * DF * 2;
    static constexpr uint32_t QK_SBO = 8 * DF * 2;
    static constexpr uint32_t V_BLOCK = C * 128;                          // 64 values x 128 keys
    static constexpr uint32_t V_BYTES = C * DV * 2;
    static constexpr uint32_t OFF_V = 0;                                   // [kStages]
    static constexpr uint32_t OFF_K = OFF_V + kStages * V_BYTES;          // [kStages]
    static constexpr uint32_t OFF_Q = OFF_K + kStages * QK_BYTES;         // [2] by unit parity
    static constexpr uint32_t OFF_L = OFF_Q + 2 * QK_BYTES;               // [kBufs][128] float row sums
    static constexpr uint32_t OFF_Z = OFF_L + kBufs * C * 4;              // [kStages] z slices
    static constexpr uint32_t OFF_BAR = OFF_Z + kStages * kZSlice;
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;          // + alignment slack
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(QK_BYTES % 1024 == 0 && V_BYTES % 1024 == 0 && OFF_L % 1024 == 0, "tile alignment");
    // TMEM: kBufs S / P buffers of 128 fp32 columns, then NO accumulators O_g.
    // Two accumulators (two O issuers) where they fit (dv = 64), one otherwise.
    static constexpr int NO = (kBufs * C + 2 * DV <= 512) ? 2 : 1;
    static constexpr uint32_t COL_S = 0, COL_O = kBufs * C;
    static constexpr uint32_t TMEM_COLS = 512;
    static_assert(COL_O + NO * DV <= TMEM_COLS, "tensor memory");
    static constexpr uint32_t ID_S = idesc_bf16_f32(128, C, false, false);
    static constexpr uint32_t ID_O = idesc_bf16_f32(128, DV, false, true);
    static constexpr int NFT = feature_tiles(DF);                         // virtual steps of a unit
};

enum {
    QB_FULL0, QB_FULL1, QB_FULL2, QB_FULL3,     // TMA: stage s (and the unit's Q) landed
    QB_EMPTY0, QB_EMPTY1, QB_EMPTY2, QB_EMPTY3, // O issuer commit: stage s read
    QB_SF0, QB_SF1, QB_SF2,                     // S issuer commit: S of buffer b ready (or buffer b free)
    QB_PF0,                                     // [kBufs][2] A group b -> O issuer og: P of buffer b
                                                // written for a step of O issuer og (step % NO)
    QB_PF_END = QB_PF0 + 2 * kBufs - 1,
    QB_OB0, QB_OB1, QB_OB2,                     // O issuer commit: P of buffer b consumed
    QB_OF,                                      // every O issuer commits once: a unit's O complete
    QB_OE,                                      // every A thread: O read out, row sums read
    QB_QE0, QB_QE1,                             // S issuer commit: Q buffer p no longer read
    QB_L,                                       // every A thread: its group's row sums written
    QB_NUM
};
static_assert(kStages == 4 && kBufs == 3, "barrier table");
static_assert(8 * QB_NUM + 8 <= 256, "barrier area");

struct QuadCtx {
    uint32_t sbase;
    uint64_t* bars;
    float* lsum;                                // [kBufs][128]
    volatile int* abort_flag;
    unsigned* status;
    int N, BH, nqt, nunits;
    int R;                                      // query tiles per chunk
    int nch;                                    // chunks per sequence
    const float* dlog;                          // decay: [BH][nqt] log2 prefix of gamma, or nullptr
    const float* zpre;                          // [BH][nch-1][NFT*128] z of each chunk's start state
};

__device__ __forceinline__ bool qwait(const QuadCtx& cx, int bar, uint32_t parity) {
    return mbar_wait(&cx.bars[bar], parity, cx.abort_flag, cx.status);
}

// Units longest first: query tiles from the last, so that the short units of
// the first chunk come at the end.
__device__ __forceinline__ void unit_of(const QuadCtx& cx, int u, int& qt, int& bh) {
    qt = cx.nqt - 1 - u / cx.BH;
    bh = u % cx.BH;
}

// Steps of the unit of query tile qt: `nvirt` virtual steps (the state of the
// chunk's start, one per feature tile; none in the first chunk), then the key
// tiles kt0..qt of its chunk.
struct UnitSteps {
    int ch, nvirt, kt0, nsteps;
};
template <int NFT>
__device__ __forceinline__ UnitSteps unit_steps(const QuadCtx& cx, int qt) {
    UnitSteps s;
    s.ch = qt / cx.R;
    s.nvirt = s.ch > 0 ? NFT : 0;
    s.kt0 = s.ch * cx.R;
    s.nsteps = s.nvirt + qt - s.kt0 + 1;
    return s;
}

// After an abort, wait (bounded) for the last asynchronous completion this
// thread is responsible for, so nothing lands in shared memory after exit.
__device__ __forceinline__ void quad_drain(const QuadCtx& cx, uint64_t* bar, uint32_t parity) {
    if (!*cx.abort_flag || bar == nullptr) return;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity) && global_ns() - t0 < kWaitLimitNs) {}
}

// ------------------------------------------------------------------ TMA producer (warp 0, lane 0)
template <int DF, int DV>
__device__ __forceinline__ void quad_producer(const QuadCtx& cx, const CUtensorMap* tq, const CUtensorMap* tk,
                                              const CUtensorMap* tv, const CUtensorMap* tp) {
    using L = QuadLayout<DF, DV>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int qt, bh;
        unit_of(cx, u, qt, bh);
        const UnitSteps us = unit_steps<L::NFT>(cx, qt);
        for (int i = 0; i < us.nsteps; ++i, ++step) {
            const int s = step % kStages;
            if (step >= kStages && !qwait(cx, QB_EMPTY0 + s, ((step / kStages) - 1) & 1)) { quad_drain(cx, last, lastp); return; }
            uint64_t* full = &cx.bars[QB_FULL0 + s];
            const int p = k_unit & 1;
            const bool virt = i < us.nvirt;
            uint32_t bytes = L::QK_BYTES + L::V_BYTES + (virt ? kZSlice : 0);
            if (i == 0) {
                // The unit's Q tile goes to the buffer of its parity once the S MMAs
                // of the unit two back are done with it; it lands with this stage.
                if (k_unit >= 2 && !qwait(cx, QB_QE0 + p, ((k_unit >> 1) - 1) & 1)) { quad_drain(cx, last, lastp); return; }
                bytes += L::QK_BYTES;
            }
            mbar_expect_tx(full, bytes);
            if (i == 0) tma_load_3d(cx.sbase + L::OFF_Q + p * L::QK_BYTES, tq, full, 0, qt * C, bh);
            if (virt) {
                // Virtual step: a copy of the Q tile in the K slot (the A warps form
                // phi(q) from it), the state tile of features [128 i, 128 i + 128)
                // in the V slot and the matching z slice.
                const int state = bh * (cx.nch - 1) + us.ch - 1;
                tma_load_3d(cx.sbase + L::OFF_K + s * L::QK_BYTES, tq, full, 0, qt * C, bh);
#pragma unroll
                for (int h = 0; h < DV / 64; ++h)
                    tma_load_3d(cx.sbase + L::OFF_V + s * L::V_BYTES + h * L::V_BLOCK, tp, full, 64 * h, C * i, state);
                bulk_load(cx.sbase + L::OFF_Z + s * kZSlice, cx.zpre + ((size_t)state * L::NFT + i) * 128, kZSlice, full);
            } else {
                const int kt = us.kt0 + (i - us.nvirt);
                tma_load_3d(cx.sbase + L::OFF_K + s * L::QK_BYTES, tk, full, 0, kt * C, bh);
#pragma unroll
                for (int h = 0; h < DV / 64; ++h)
                    tma_load_3d(cx.sbase + L::OFF_V + s * L::V_BYTES + h * L::V_BLOCK, tv, full, 64 * h, kt * C, bh);
            }
            last = full;
            lastp = (step / kStages) & 1;
        }
    }
    quad_drain(cx, last, lastp);
}

// A of one slice (16 keys, from column j_base) of row i: P = bf16(1 + S + S^2/2),
// times the decay weight w of the tile pair (DECAY), masked past i on the
// diagonal tile, with the row sum accumulated in fp32.
template <bool DECAY>
__device__ __forceinline__ void quad_slice(const float* sv, uint32_t* pw, int j_base, int i, bool diag, float w,
                                           float& l0, float& l1) {
#pragma unroll
    for (int m = 0; m < 8; ++m) {
        float a0, a1;
        taylor_pair(sv[2 * m], sv[2 * m + 1], a0, a1);
        if constexpr (DECAY) {
            a0 *= w;                             // the tile pair's decay weight
            a1 *= w;
        }
        if (diag) {
            const int j0 = j_base + 2 * m;
            a0 = j0 <= i ? a0 : 0.0f;
            a1 = j0 + 1 <= i ? a1 : 0.0f;
        }
        add_pair(l0, l1, a0, a1);
        pw[m] = pack_bf16x2(a0, a1);
    }
}

// ------------------------------------------------------------------ virtual steps: phi(q) slices
// x_A of a query row held as packed bf16 pairs xw (two per word, lower index in
// the low half), with x_DF = 1 the constant: unpacked where used, which keeps
// the row in d'/2 registers.
template <int DF, int A>
__device__ __forceinline__ float xval(const uint32_t* xw) {
    if constexpr (A == DF) return 1.0f;
    else if constexpr (A & 1) return __uint_as_float(xw[A / 2] & 0xFFFF0000u);
    else return __uint_as_float(xw[A / 2] << 16);
}

// Folded feature F of the row: x_a x_b times its coefficient (compile-time pair).
template <int DF, int F>
__device__ __forceinline__ float phi_f(const uint32_t* xw) {
    constexpr FeatPair fp = feat_pair(DF, F);
    return (xval<DF, fp.a>(xw) * xval<DF, fp.b>(xw)) * fp.coef;
}

// Features F0 .. F0+15 of the row as 8 bf16 pairs into pw; their fp32 values
// dotted with the z slice (16 floats at shared address zaddr) accumulate into l.
template <int DF, int F0, int... E>
__device__ __forceinline__ void phi_piece16(const uint32_t* xw, uint32_t zaddr, uint32_t* pw, float& l0, float& l1,
                                            std::integer_sequence<int, E...>) {
    const float f[16] = {phi_f<DF, F0 + E>(xw)...};
#pragma unroll
    for (int m4 = 0; m4 < 4; ++m4) {
        const uint4 zz = ld_shared_v4(zaddr + 16 * m4);
        l0 = fmaf(f[4 * m4], __uint_as_float(zz.x), l0);
        l1 = fmaf(f[4 * m4 + 1], __uint_as_float(zz.y), l1);
        l0 = fmaf(f[4 * m4 + 2], __uint_as_float(zz.z), l0);
        l1 = fmaf(f[4 * m4 + 3], __uint_as_float(zz.w), l1);
    }
#pragma unroll
    for (int m = 0; m < 8; ++m) pw[m] = pack_bf16x2(f[2 * m], f[2 * m + 1]);
}

template <int DF, int F0, int K, int KMAX>
__device__ __forceinline__ void phi_pieces(const uint32_t* xw, uint32_t zaddr, uint32_t pcol, float& l0, float& l1) {
    if constexpr (K < KMAX) {
        uint32_t pw[8];
        phi_piece16<DF, F0 + 16 * K>(xw, zaddr + 64 * K, pw, l0, l1, std::make_integer_sequence<int, 16>{});
        tmem_st8(pcol + 8 * K, pw);
        phi_pieces<DF, F0, K + 1, KMAX>(xw, zaddr, pcol, l0, l1);
    }
}

// Features [128 V, 128 V + 128) of the row into P (TMEM columns `pcol`..+63, two
// features per column, lower feature in the low half), for the runtime tile v.
template <int DF, int V, int VMAX>
__device__ __forceinline__ void phi_slice(int v, const uint32_t* xw, uint32_t zaddr, uint32_t pcol, float& l0,
                                          float& l1) {
    if constexpr (V < VMAX) {
        if (v == V) {
            phi_pieces<DF, 128 * V, 0, 8>(xw, zaddr, pcol, l0, l1);
            return;
        }
        phi_slice<DF, V + 1, VMAX>(v, xw, zaddr, pcol, l0, l1);
    }
}

// One virtual step of one query row, as a call of its own: its fully unrolled
// feature code would otherwise share the register budget of the A warps' loop
// (and spill there). Returns the increments of the two row-sum accumulators.
template <int DF>
struct QRow {
    uint32_t w[DF / 2];                          // q as bf16 pairs
};
template <int DF, int NFT>
__device__ __noinline__ float2 virtual_step(int v, QRow<DF> q, uint32_t zaddr, uint32_t pcol) {
    float l0 = 0.0f, l1 = 0.0f;
    phi_slice<DF, 0, NFT>(v, q.w, zaddr, pcol, l0, l1);
    return make_float2(l0, l1);
}

// ------------------------------------------------------------------ A warps (4-15)
// Group g (of kBufs) forms P for the steps with step % kBufs == g, in S / P
// buffer g, and keeps the row sums l of its steps. At the end of a unit the
// groups pool their row sums through shared memory and write y = O / l, group g
// for the 32-column blocks h = g, g + kBufs, ... Thread = query row i = TMEM
// lane (wq = lane quadrant).
template <int DF, int DV, bool DECAY>
__device__ __forceinline__ void quad_rows(const QuadCtx& cx, uint32_t tmem, int g, int wq, int lane,
                                          __nv_bfloat16* __restrict__ y) {
    using L = QuadLayout<DF, DV>;
    const int i = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t sb = tmem + lane_off + L::COL_S + g * C;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int qt, bh;
        unit_of(cx, u, qt, bh);
        const UnitSteps us = unit_steps<L::NFT>(cx, qt);
        const int step0 = step;
        float l0 = 0.0f, l1 = 0.0f;
        for (int j = 0; j < us.nsteps; ++j, ++step) {
            if (step % kBufs != g) continue;
            if (!qwait(cx, QB_SF0 + g, (step / kBufs) & 1)) return;
            tc_fence_after();
            if (j < us.nvirt) {
                // Virtual step j: P = phi(q_i) over feature tile j, from the Q copy and
                // the z slice of this step's stage (waiting for the stage's load makes
                // them visible to this thread).
                const int s = step % kStages;
                if (!qwait(cx, QB_FULL0 + s, (step / kStages) & 1)) return;
                QRow<DF> qr;                              // q_i as bf16 pairs
                const uint32_t qrow = cx.sbase + L::OFF_K + s * L::QK_BYTES;
#pragma unroll
                for (int c = 0; c < DF / 8; ++c) {
                    const uint32_t o = i * (DF * 2) + 16 * c;
                    const uint32_t phys = o ^ (((o >> 7) & (L::QK_SWIZZLE / 16 - 1)) << 4);
                    const uint4 w4 = ld_shared_v4(qrow + phys);
                    qr.w[4 * c] = w4.x;
                    qr.w[4 * c + 1] = w4.y;
                    qr.w[4 * c + 2] = w4.z;
                    qr.w[4 * c + 3] = w4.w;
                }
                const float2 dl = virtual_step<DF, L::NFT>(j, qr, cx.sbase + L::OFF_Z + s * kZSlice, sb);
                l0 += dl.x;
                l1 += dl.y;
            } else {
                const int kt = us.kt0 + (j - us.nvirt);
                const bool diag = kt == qt;      // keys j > i of the diagonal tile are masked
                // Coarse decay: key tile kt reaches query tile qt scaled by the product
                // of gamma over tiles kt+1..qt = 2^(L[qt] - L[kt]).
                const float w = DECAY ? exp2f(cx.dlog[(size_t)bh * cx.nqt + qt] - cx.dlog[(size_t)bh * cx.nqt + kt]) : 1.0f;
                // Slice c reads S columns 16c..16c+15 and writes P columns 8c..8c+7,
                // which overlay S columns already read; the next slice's load is in
                // flight while a slice is computed.
                float s0[16], s1[16];
                uint32_t pw[8];
                tmem_ld16(sb, s0);
                tmem_ld_wait();
#pragma unroll 1
                for (int c2 = 0; c2 < 4; ++c2) {
                    tmem_ld16(sb + 32 * c2 + 16, s1);
                    quad_slice<DECAY>(s0, pw, 32 * c2, i, diag, w, l0, l1);
                    tmem_st8(sb + 16 * c2, pw);
                    tmem_ld_wait();
                    if (c2 < 3) tmem_ld16(sb + 32 * c2 + 32, s0);
                    quad_slice<DECAY>(s1, pw, 32 * c2 + 16, i, diag, w, l0, l1);
                    tmem_st8(sb + 16 * c2 + 8, pw);
                    if (c2 < 3) tmem_ld_wait();
                }
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&cx.bars[QB_PF0 + 2 * g + step % L::NO]);
        }
        // Row sums: publish this group's once every group has read the previous
        // unit's (they arrive on OE only after reading them), then pool.
        if (k_unit >= 1 && !qwait(cx, QB_OE, (k_unit - 1) & 1)) return;
        cx.lsum[g * C + i] = l0 + l1;
        mbar_arrive(&cx.bars[QB_L]);
        if (!qwait(cx, QB_L, k_unit & 1)) return;
        float lt = 0.0f;
#pragma unroll
        for (int gg = 0; gg < kBufs; ++gg) lt += cx.lsum[gg * C + i];
        const float inv = 1.0f / lt;             // l >= 1/2 for every real row
        if (!qwait(cx, QB_OF, k_unit & 1)) return;
        tc_fence_after();
        // With two accumulators, O_b holds the unit's steps of parity b, if any.
        const int nsteps = us.nsteps;
        const bool has0 = L::NO == 1 || nsteps >= 2 || (step0 & 1) == 0;
        const bool has1 = L::NO == 2 && (nsteps >= 2 || (step0 & 1) == 1);
        const int tok = qt * C + i;
        uint4* yp = reinterpret_cast<uint4*>(y + ((size_t)bh * cx.N + (tok < cx.N ? tok : 0)) * DV);
        const uint32_t ob = tmem + lane_off + L::COL_O;
#pragma unroll 1
        for (int h = g; h < DV / 32; h += kBufs) {
            float o[32], o1[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0.0f, o1[e] = 0.0f;
            if (has0) {
                tmem_ld16(ob + 32 * h, o);
                tmem_ld16(ob + 32 * h + 16, o + 16);
            }
            if (has1) {
                tmem_ld16(ob + DV + 32 * h, o1);
                tmem_ld16(ob + DV + 32 * h + 16, o1 + 16);
            }
            tmem_ld_wait();
            const size_t y_at = ((size_t)bh * cx.N + tok) * DV + 32 * h;
            if (tok < cx.N && in_bounds(y_at + 31, (size_t)cx.BH * cx.N * DV, cx.status)) {
#pragma unroll
                for (int p8 = 0; p8 < 4; ++p8) {
                    float t8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t8[e] = (o[8 * p8 + e] + o1[8 * p8 + e]) * inv;
                    yp[4 * h + p8] = pack_bf16x8(t8);
                }
            }
        }
        tc_fence_before();
        mbar_arrive(&cx.bars[QB_OE]);            // O may be overwritten by the next unit
    }
}

// ------------------------------------------------------------------ issuers
// S = Q K^T of every intra step (warp 1, lane 0), into S buffer step % kBufs;
// a virtual step only takes the buffer (its P comes from the A warps).
template <int DF, int DV>
__device__ __forceinline__ void quad_s_issuer(const QuadCtx& cx, uint32_t tmem) {
    using L = QuadLayout<DF, DV>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int qt, bh;
        unit_of(cx, u, qt, bh);
        const UnitSteps us = unit_steps<L::NFT>(cx, qt);
        const int p = k_unit & 1;
        const uint64_t dq = smem_desc_swizzled(cx.sbase + L::OFF_Q + p * L::QK_BYTES, 16, L::QK_SBO, L::QK_SWIZZLE);
        for (int j = 0; j < us.nsteps; ++j, ++step) {
            const int s = step % kStages, b = step % kBufs;
            if (!qwait(cx, QB_FULL0 + s, (step / kStages) & 1)) { quad_drain(cx, last, lastp); return; }
            if (step >= kBufs && !qwait(cx, QB_OB0 + b, ((step / kBufs) - 1) & 1)) { quad_drain(cx, last, lastp); return; }
            tc_fence_after();
            if (j >= us.nvirt) {
                const uint64_t dk = smem_desc_swizzled(cx.sbase + L::OFF_K + s * L::QK_BYTES, 16, L::QK_SBO, L::QK_SWIZZLE);
#pragma unroll
                for (int jj = 0; jj < DF / 16; ++jj)    // K step of 16 = 32 bytes along the swizzled row
                    mma_bf16(tmem + L::COL_S + b * C, dq + 2 * jj, dk + 2 * jj, L::ID_S, jj > 0);
            }
            mma_commit(&cx.bars[QB_SF0 + b]);
            last = &cx.bars[QB_SF0 + b];
            lastp = (step / kBufs) & 1;
            if (j + 1 == us.nsteps) mma_commit(&cx.bars[QB_QE0 + p]);
        }
    }
    quad_drain(cx, last, lastp);
}

// O_og += P V of the steps with step % NO == og (warp 2 + og, lane 0).
template <int DF, int DV>
__device__ __forceinline__ void quad_o_issuer(const QuadCtx& cx, uint32_t tmem, int og) {
    using L = QuadLayout<DF, DV>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    const uint32_t d_tmem = tmem + L::COL_O + og * DV;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int qt, bh;
        unit_of(cx, u, qt, bh);
        const UnitSteps us = unit_steps<L::NFT>(cx, qt);
        // O is free once every A thread has read out the previous unit.
        if (k_unit >= 1 && !qwait(cx, QB_OE, (k_unit - 1) & 1)) { quad_drain(cx, last, lastp); return; }
        bool first = true;
        for (int j = 0; j < us.nsteps; ++j, ++step) {
            if (step % L::NO != og) continue;
            const int s = step % kStages, b = step % kBufs;
            // One barrier per (buffer, issuer): each is consumed in order by one
            // thread, so a waiter is never two phases ahead of it (with two
            // issuers sharing a buffer's barrier, the later one could be, and a
            // parity wait would then pass on the previous phase).
            if (!qwait(cx, QB_PF0 + 2 * b + og, (step / (kBufs * L::NO)) & 1)) { quad_drain(cx, last, lastp); return; }
            tc_fence_after();
            const uint64_t dv = smem_desc_sw128(cx.sbase + L::OFF_V + s * L::V_BYTES, L::V_BLOCK, 1024);
            const uint32_t a_tmem = tmem + L::COL_S + b * C;
#pragma unroll
            for (int jj = 0; jj < C / 16; ++jj)      // K step of 16 keys (or features) = 2048 bytes
                mma_bf16_ts(d_tmem, a_tmem + 8 * jj, dv + ((jj * 2048) >> 4), L::ID_O, (!first || jj > 0) ? 1u : 0u);
            first = false;
            mma_commit(&cx.bars[QB_EMPTY0 + s]);     // S and O of this step have read the stage
            mma_commit(&cx.bars[QB_OB0 + b]);
            last = &cx.bars[QB_OB0 + b];
            lastp = (step / kBufs) & 1;
        }
        mma_commit(&cx.bars[QB_OF]);
        last = &cx.bars[QB_OF];
        lastp = k_unit & 1;
    }
    quad_drain(cx, last, lastp);
}

template <int DF, int DV, bool DECAY>
__global__ void __launch_bounds__(kQuadThreads, 1)
la_quad_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
               const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tp,
               __nv_bfloat16* __restrict__ y, int N, int BH, int nqt, int R, int nch,
               const float* __restrict__ dlog, const float* __restrict__ zpre, unsigned* status, unsigned debug) {
    using L = QuadLayout<DF, DV>;
    extern __shared__ unsigned char quad_smem[];
    const uint32_t raw = smem_u32(quad_smem);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = quad_smem + (sbase - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + 8 * QB_NUM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BAR + 8 * QB_NUM + 4);
    const QuadCtx cx{sbase, bars, reinterpret_cast<float*>(smem + L::OFF_L), abort_flag, status, N, BH, nqt,
                     nqt * BH, R, nch, dlog, zpre};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int b = 0; b < QB_NUM; ++b) {
            uint32_t count = 1;
            if (b >= QB_PF0 && b <= QB_PF_END) count = 128;
            if (b == QB_L || b == QB_OE) count = kBufs * 128;
            if (b == QB_OF) count = L::NO;
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
    const bool skip_mma = (debug & DEBUG_SKIP_MMA) != 0;   // testing: issue nothing, every waiter times out

    if (warp == 0) {
        if (lane == 0) quad_producer<DF, DV>(cx, &tq, &tk, &tv, &tp);
    } else if (warp == 1) {
        if (lane == 0 && !skip_mma) quad_s_issuer<DF, DV>(cx, tmem);
    } else if (warp < 4) {
        if (lane == 0 && !skip_mma && warp - 2 < L::NO) quad_o_issuer<DF, DV>(cx, tmem, warp - 2);
    } else {
        quad_rows<DF, DV, DECAY>(cx, tmem, (warp - 4) >> 2, warp & 3, lane, y);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ prefix states and final state
// One CTA per (b, h, tile of 128 folded features), two CTAs per SM: D (TMEM
// lane = feature) += phi(K)^T V per step of 64 tokens, M=128 N=dv K=64, and z
// (the features' sums over tokens) in fp32 on the CUDA cores. Warp 5 (lane 0)
// loads each step's K and V by TMA into a 3-stage ring; warps 0-3 (thread =
// token t, half fh of the tile's features) read k_t from shared memory, write
// their 64 features of phi(k_t) into a double-buffered operand and add them
// to per-thread sums; warp 4 allocates TMEM and issues the MMAs. After the
// step that ends a chunk (every `snap_steps` steps, the last excepted) the
// state is written out as the start state of the next chunk: warps 0-3
// (thread = feature) read D after that step's MMAs, round it to bf16 and
// store the feature's row; z is pooled from the per-thread sums (a butterfly
// within each warp, then across the two warps of a half). At the end warps
// 0-3 write the feature's rows of the 1 + d' + d'^2 layout (or the symmetric
// one): the constant, the d' linear rows, and each folded pair x_a x_b as rows
// (a, b) and (b, a), each times 1/sqrt2 (the diagonal x_a^2 carries its
// 1/sqrt2 already).
constexpr int kStateThreads = 192;
constexpr int CS = 64;               // tokens per MMA step
constexpr int kSStages = 3;
constexpr int kL2Ahead = 8;          // steps whose K, V tiles are prefetched into L2 ahead of their load

// Folded feature F of a token whose inputs are in fp32 registers (x[DF] the constant).
template <int DF, int F>
__device__ __forceinline__ float phi_fx(const float* x) {
    constexpr FeatPair fp = feat_pair(DF, F);
    return (x[fp.a] * x[fp.b]) * fp.coef;
}

// phi(k) of one token for 8 consecutive features from F0 (compile-time pairs),
// scaled by u, as bf16 into the operand and in fp32 into the running sums.
template <int DF, int F0, int... E>
__device__ __forceinline__ uint4 state_piece(const float* x, float u, float* zacc, std::integer_sequence<int, E...>) {
    const float f8[8] = {(phi_fx<DF, F0 + E>(x) * u)...};
#pragma unroll
    for (int e = 0; e < 8; ++e) zacc[e] += f8[e];
    return pack_bf16x8(f8);
}

template <int DF, int F0, int... J>
__device__ __forceinline__ void state_phi_half_impl(const float* x, float u, float* zacc, uint32_t row, uint32_t sbo,
                                                    std::integer_sequence<int, J...>) {
    ((st_shared_v4(row + J * sbo, state_piece<DF, F0 + 8 * J>(x, u, zacc + 8 * J, std::make_integer_sequence<int, 8>{}))), ...);
}

// Features [64 H, 64 H + 64) for the selector sel == H (H < HMAX).
template <int DF, int H, int HMAX>
__device__ __forceinline__ void state_phi_half(int sel, const float* x, float u, float* zacc, uint32_t row,
                                               uint32_t sbo) {
    if constexpr (H < HMAX) {
        if (sel == H) {
            state_phi_half_impl<DF, 64 * H>(x, u, zacc, row, sbo, std::make_integer_sequence<int, 8>{});
            return;
        }
        state_phi_half<DF, H + 1, HMAX>(sel, x, u, zacc, row, sbo);
    }
}

template <int DF, int DV>
struct StateLayout {
    static constexpr int DS = sym_feature_dim(DF);
    static constexpr int NFT = feature_tiles(DF);
    static constexpr uint32_t A_BYTES = 128 * CS * 2;    // phi(K)^T: M = feature, K = token, MN-major
    static constexpr uint32_t A_LBO = (128 / 8) * 128, A_SBO = 128;
    static constexpr int K_SWIZZLE = DF * 2;             // K tile: rows of d' bf16, swizzled
    static constexpr uint32_t K_BYTES = CS * DF * 2;
    static constexpr uint32_t V_BLOCK = CS * 128;        // 64 values x 64 tokens, 128-byte swizzle
    static constexpr uint32_t V_BYTES = (DV / 64) * V_BLOCK;
    static constexpr uint32_t OFF_A = 0;                 // [2]
    static constexpr uint32_t OFF_V = 2 * A_BYTES;       // [kSStages]
    static constexpr uint32_t OFF_K = OFF_V + kSStages * V_BYTES;   // [kSStages]
    static constexpr uint32_t OFF_Z = OFF_K + kSStages * K_BYTES;   // [2 poolings][2 warps][128] floats
    static constexpr uint32_t OFF_BAR = OFF_Z + 2 * 2 * 128 * 4;
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 128 + 1024;   // + alignment slack
    static_assert(2 * SMEM_BYTES <= 226 * 1024, "two CTAs per SM");
    static_assert(OFF_K % 1024 == 0 && K_BYTES % 512 == 0, "tile alignment");
    static_assert(NFT <= 5, "feature tiles dispatched in la_prefix_kernel");
    static constexpr uint32_t TMEM_COLS = DV;
    static constexpr uint32_t ID = idesc_bf16_f32(128, DV, true, true);
};

enum {
    SB_FULL0, SB_FULL1, SB_FULL2,     // TMA: stage s landed
    SB_EMPTY0, SB_EMPTY1, SB_EMPTY2,  // MMA commit: stage s read
    SB_PHI0, SB_PHI1,                 // builders: phi operand b written
    SB_AFREE0, SB_AFREE1,             // MMA commit: phi operand b read
    SB_SNAP,                          // MMA commit: the state at a chunk boundary is complete
    SB_SNAPF,                         // builders: that state has been read
    SB_DONE,                          // MMA commit: the final state is complete
    SB_ZW,                            // builders: their partial z sums of a pooling are in shared memory
    SB_NUM
};
static_assert(8 * SB_NUM + 8 <= 128, "barrier area");

// z of the tile's feature `tid` over the tokens summed in zacc since the last
// pooling (number k): each warp's 32 tokens by a butterfly (lane l ends with
// features 2l, 2l + 1 of its half), then the two warps of a half through
// shared memory (buffer k mod 2, so that pooling k+1 never overwrites what a
// slow thread still reads of pooling k: every thread has arrived for k+1 only
// after reading k). All four builder warps call it together; the hand-off is a
// bounded mbarrier wait, so a warp that gave up cannot stall the others.
template <int DF, int DV>
__device__ __forceinline__ bool pool_z(float* zacc, int warp, int lane, int tid, float* zred, int k, uint64_t* bar,
                                       volatile int* abort_flag, unsigned* status, float& out) {
    float z[64];
#pragma unroll
    for (int e = 0; e < 64; ++e) z[e] = zacc[e];
#pragma unroll
    for (int o = 16, n = 64; o >= 1; o >>= 1, n >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int e = 0; e < n / 2; ++e) {
            const float send = upper ? z[e] : z[e + n / 2];
            const float keep = upper ? z[e + n / 2] : z[e];
            z[e] = keep + __shfl_xor_sync(0xffffffffu, send, o);
        }
    }
    const int half = warp >> 1, part = warp & 1;
    float* zb = zred + (k & 1) * 256;
    zb[part * 128 + 64 * half + 2 * lane] = z[0];
    zb[part * 128 + 64 * half + 2 * lane + 1] = z[1];
    mbar_arrive(bar);
    if (!mbar_wait(bar, k & 1, abort_flag, status)) return false;
    out = zb[tid] + zb[128 + tid];
    return true;
}

template <int DF, int DV, bool DECAY>
__global__ void __launch_bounds__(kStateThreads, 2)
la_prefix_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                 float* __restrict__ S, float* __restrict__ z, __nv_bfloat16* __restrict__ spre,
                 float* __restrict__ zpre, int N, int snap_steps, int nch, int packed,
                 const float* __restrict__ dlog, unsigned* status, unsigned debug) {
    using L = StateLayout<DF, DV>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + 8 * SB_NUM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BAR + 8 * SB_NUM + 4);
    float* zred = reinterpret_cast<float*>(smem + L::OFF_Z);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / L::NFT;
    const int ft = blockIdx.x % L::NFT;
    const int f0 = ft * 128;
    const int nsteps = (N + CS - 1) / CS;
    const int nqt = (N + 127) / 128;                      // 128-token decay tiles
    const size_t n_heads = gridDim.x / L::NFT;            // extents for the index checks
    // A chunk boundary follows step c when (c + 1) is a multiple of snap_steps
    // and another step comes after it.
    auto boundary_after = [&](int c) { return (c + 1) % snap_steps == 0 && c + 1 < nsteps; };

    if (tid == 0) {
        for (int b = 0; b < SB_NUM; ++b)
            mbar_init(&bars[b], (b == SB_PHI0 || b == SB_PHI1 || b == SB_SNAPF || b == SB_ZW) ? 128 : 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 4) tmem_alloc(tmem_slot, L::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        const int t = tid & (CS - 1), fh = tid / CS;
        const uint32_t arow = sbase + L::OFF_A + (t & 7) * 16 + (t >> 3) * L::A_LBO + 8 * fh * L::A_SBO;
        const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);   // lane = feature f0 + tid
        const int f = f0 + tid;
        float zacc[64];
#pragma unroll
        for (int e = 0; e < 64; ++e) zacc[e] = 0.0f;
        float zrun = 0.0f;                                 // z of feature f over the pooled steps
        int snaps = 0, pools = 0;
        bool ok = true;
        for (int c = 0; ok && c < nsteps; ++c) {
            const int s = c % kSStages, b = c & 1;
            if (!mbar_wait(&bars[SB_FULL0 + s], (c / kSStages) & 1, abort_flag, status)) { ok = false; break; }
            if (c >= 2 && !mbar_wait(&bars[SB_AFREE0 + b], ((c >> 1) - 1) & 1, abort_flag, status)) { ok = false; break; }
            // k of token t from the swizzled K tile (rows past N read as 0).
            float x[DF + 1];
            const uint32_t krow = sbase + L::OFF_K + s * L::K_BYTES;
#pragma unroll
            for (int j = 0; j < DF / 8; ++j) {
                const uint32_t o = t * (DF * 2) + 16 * j;
                const uint32_t phys = o ^ (((o >> 7) & (L::K_SWIZZLE / 16 - 1)) << 4);
                const uint4 w4 = ld_shared_v4(krow + phys);
                const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * j + 2 * e] = __uint_as_float(wd[e] << 16);
                    x[8 * j + 2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u);
                }
            }
            const int tok = c * CS + t;
            x[DF] = tok < N ? 1.0f : 0.0f;
            // Coarse decay: token t's contribution to the final state is scaled by the
            // product of gamma over the 128-token tiles after its own.
            const float u = DECAY ? (tok < N ? exp2f(dlog[(size_t)bh * nqt + nqt - 1] - dlog[(size_t)bh * nqt + tok / 128]) : 0.0f)
                                  : 1.0f;
            state_phi_half<DF, 0, 2 * L::NFT>(2 * ft + fh, x, u, zacc, arow + b * L::A_BYTES, L::A_SBO);
            fence_proxy_async_smem();
            mbar_arrive(&bars[SB_PHI0 + b]);
            // The state at the boundary after the previous step: once that step's MMAs
            // are done, feature f's row in bf16 to the workspace.
            if (c >= 1 && boundary_after(c - 1)) {
                if (!mbar_wait(&bars[SB_SNAP], snaps & 1, abort_flag, status)) { ok = false; break; }
                tc_fence_after();
                const int chunk = (c * CS) / (snap_steps * CS);        // the chunk that starts here
                const size_t row = ((size_t)bh * (nch - 1) + chunk - 1) * (L::NFT * 128) + f;
                const bool row_ok = in_bounds(row, n_heads * (nch - 1) * (L::NFT * 128), status);
                uint4* dst = reinterpret_cast<uint4*>(spre + row * DV);
#pragma unroll 1
                for (int m = 0; m < DV / 16; ++m) {
                    float r[16];
                    tmem_ld16(taddr + 16 * m, r);
                    tmem_ld_wait();
                    if (row_ok) {
                        dst[2 * m] = pack_bf16x8(r);
                        dst[2 * m + 1] = pack_bf16x8(r + 8);
                    }
                }
                tc_fence_before();
                mbar_arrive(&bars[SB_SNAPF]);
                ++snaps;
            }
            // z of the tokens before the boundary after this step.
            if (boundary_after(c)) {
                float zp;
                if (!pool_z<DF, DV>(zacc, warp, lane, tid, zred, pools++, &bars[SB_ZW], abort_flag, status, zp)) {
                    ok = false;
                    break;
                }
                zrun += zp;
#pragma unroll
                for (int e = 0; e < 64; ++e) zacc[e] = 0.0f;
                const int chunk = ((c + 1) * CS) / (snap_steps * CS);
                const size_t at = ((size_t)bh * (nch - 1) + chunk - 1) * (L::NFT * 128) + f;
                if (in_bounds(at, n_heads * (nch - 1) * (L::NFT * 128), status)) zpre[at] = zrun;
            }
        }
        // Epilogue: thread = feature f (TMEM lane), rows of the full or the symmetric layout.
        if (ok) {
            float zp;
            ok = pool_z<DF, DV>(zacc, warp, lane, tid, zred, pools++, &bars[SB_ZW], abort_flag, status, zp);
            zrun += zp;
        }
        if (ok && S != nullptr && mbar_wait(&bars[SB_DONE], 0, abort_flag, status)) {
            tc_fence_after();
            const FeatPair fp = feat_pair(DF, f < L::DS ? f : 0);
            const int ia = fp.a, ib = fp.b;
            // Full layout: the constant, the d' linear rows, and each folded pair in
            // rows (a, b) and (b, a). Symmetric layout: the folded row itself.
            const int D = packed ? L::DS : feature_dim(DF);
            int r0 = 0, r1 = -1;
            float coef = 1.0f;
            if (packed || f <= DF) {
                r0 = f;
            } else {
                r0 = 1 + DF + ia * DF + ib;
                if (ia != ib) { r1 = 1 + DF + ib * DF + ia; coef = kSqrtHalf; }
            }
            const size_t hb = static_cast<size_t>(bh);
#pragma unroll 1
            for (int m = 0; m < DV / 16; ++m) {
                float r[16];
                tmem_ld16(taddr + 16 * m, r);
                tmem_ld_wait();
                if (f >= L::DS || !in_bounds((hb * D + (r1 >= 0 ? max(r0, r1) : r0)) * DV + 16 * m + 15,
                                             n_heads * D * DV, status))
                    continue;
                float4* row0 = reinterpret_cast<float4*>(S + (hb * D + r0) * DV + 16 * m);
                float4* row1 = reinterpret_cast<float4*>(S + (hb * D + (r1 >= 0 ? r1 : r0)) * DV + 16 * m);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float4 val = make_float4(r[4 * e] * coef, r[4 * e + 1] * coef, r[4 * e + 2] * coef,
                                                   r[4 * e + 3] * coef);
                    row0[e] = val;
                    if (r1 >= 0) row1[e] = val;
                }
            }
            if (f < L::DS && in_bounds(hb * D + (r1 >= 0 ? max(r0, r1) : r0), n_heads * D, status)) {
                z[hb * D + r0] = zrun * coef;
                if (r1 >= 0) z[hb * D + r1] = zrun * coef;
            }
        }
    } else if (warp == 4) {
        if (lane == 0 && !(debug & DEBUG_SKIP_MMA)) {
            uint64_t* last = nullptr;
            uint32_t lastp = 0;
            int snaps = 0;
            for (int c = 0; c < nsteps; ++c) {
                const int s = c % kSStages, b = c & 1;
                if (!mbar_wait(&bars[SB_PHI0 + b], (c >> 1) & 1, abort_flag, status)) break;
                if (!mbar_wait(&bars[SB_FULL0 + s], (c / kSStages) & 1, abort_flag, status)) break;
                // The state at a boundary is read before the next step adds to it.
                if (c >= 1 && boundary_after(c - 1) && !mbar_wait(&bars[SB_SNAPF], (snaps - 1) & 1, abort_flag, status))
                    break;
                tc_fence_after();
                const uint64_t da = smem_desc(sbase + L::OFF_A + b * L::A_BYTES, L::A_LBO, L::A_SBO);
                const uint64_t dv = smem_desc_sw128(sbase + L::OFF_V + s * L::V_BYTES, L::V_BLOCK, 1024);
#pragma unroll
                for (int j = 0; j < CS / 16; ++j)
                    mma_bf16(tmem, da + ((j * 2 * L::A_LBO) >> 4), dv + ((j * 2048) >> 4), L::ID,
                             (c > 0 || j > 0) ? 1u : 0u);
                mma_commit(&bars[SB_EMPTY0 + s]);
                mma_commit(&bars[SB_AFREE0 + b]);
                last = &bars[SB_AFREE0 + b];
                lastp = (c >> 1) & 1;
                if (boundary_after(c)) {
                    mma_commit(&bars[SB_SNAP]);
                    last = &bars[SB_SNAP];
                    lastp = snaps & 1;
                    ++snaps;
                }
            }
            if (!*abort_flag) {
                mma_commit(&bars[SB_DONE]);
            } else if (last != nullptr) {
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(last, lastp) && global_ns() - t0 < kWaitLimitNs) {}
            }
        }
    } else if (lane == 0) {
        // TMA: step c into stage c mod 3 once the MMAs of step c - 3 are done with it.
        // A load that misses L2 takes ~2.4k cycles here, longer than three steps of
        // work, so the tiles kL2Ahead steps ahead are first prefetched into L2.
        uint64_t* last = nullptr;
        uint32_t lastp = 0;
        for (int c = 0; c < kL2Ahead && c < nsteps; ++c) {
            tma_prefetch_3d(&tk, 0, c * CS, bh);
#pragma unroll
            for (int h = 0; h < DV / 64; ++h) tma_prefetch_3d(&tv, 64 * h, c * CS, bh);
        }
        for (int c = 0; c < nsteps; ++c) {
            const int s = c % kSStages;
            if (c + kL2Ahead < nsteps) {
                tma_prefetch_3d(&tk, 0, (c + kL2Ahead) * CS, bh);
#pragma unroll
                for (int h = 0; h < DV / 64; ++h) tma_prefetch_3d(&tv, 64 * h, (c + kL2Ahead) * CS, bh);
            }
            if (c >= kSStages && !mbar_wait(&bars[SB_EMPTY0 + s], ((c / kSStages) - 1) & 1, abort_flag, status)) break;
            uint64_t* full = &bars[SB_FULL0 + s];
            mbar_expect_tx(full, L::K_BYTES + L::V_BYTES);
            tma_load_3d(sbase + L::OFF_K + s * L::K_BYTES, &tk, full, 0, c * CS, bh);
#pragma unroll
            for (int h = 0; h < DV / 64; ++h)
                tma_load_3d(sbase + L::OFF_V + s * L::V_BYTES + h * L::V_BLOCK, &tv, full, 64 * h, c * CS, bh);
            last = full;
            lastp = (c / kSStages) & 1;
        }
        if (*abort_flag && last != nullptr) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(last, lastp) && global_ns() - t0 < kWaitLimitNs) {}
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// Coarse decay: L[bh][c] = sum over tiles c' <= c of log2 gamma[bh][c'], so that
// the product of gamma over tiles a+1..b is 2^(L[b] - L[a]).
__global__ void decay_log2_prefix_kernel(const float* __restrict__ gamma, float* __restrict__ dlog, int BH,
                                         int nqt) {
    const int bh = blockIdx.x * blockDim.x + threadIdx.x;
    if (bh >= BH) return;
    float acc = 0.0f;
    for (int c = 0; c < nqt; ++c) {
        acc += log2f(gamma[(size_t)bh * nqt + c]);
        dlog[(size_t)bh * nqt + c] = acc;
    }
}

// Chunks of `chunk` tokens (a multiple of 128; 0 or >= N: one chunk, the
// quadratic form) and the workspace bytes their start states take:
// bf16 S [BH][nch-1][NFT*128][DV], then fp32 z [BH][nch-1][NFT*128].
struct ChunkCfg {
    int R, nch;
    size_t s_bytes, z_bytes;
};
ChunkCfg chunk_cfg(int B, int H, int N, int d_feat, int d_v, int chunk) {
    ChunkCfg c;
    const int nqt = (N + C - 1) / C;
    c.R = (chunk <= 0 || chunk >= N) ? nqt : chunk / C;
    c.nch = (nqt + c.R - 1) / c.R;
    const size_t states = (size_t)B * H * (c.nch - 1) * feature_tiles(d_feat) * 128;
    c.s_bytes = states * d_v * 2;
    c.z_bytes = states * 4;
    return c;
}

template <int DF, int DV>
cudaError_t launch_quad_typed(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    const int BH = a.B * a.H;
    const int nqt = (a.N + C - 1) / C;
    const long long nunits = (long long)nqt * BH;
    if (nunits > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    const bool decay = a.gamma != nullptr;
    const ChunkCfg cc = chunk_cfg(a.B, a.H, a.N, DF, DV, decay ? 0 : a.chunk);
    using SL = StateLayout<DF, DV>;
    bf* spre = nullptr;
    float* zpre = nullptr;
    if (cc.nch > 1) {
        if (a.workspace == nullptr || a.ws_bytes < cc.s_bytes + cc.z_bytes) return cudaErrorInvalidValue;
        spre = static_cast<bf*>(a.workspace);
        zpre = reinterpret_cast<float*>(static_cast<unsigned char*>(a.workspace) + cc.s_bytes);
    }
    const float* dlog = nullptr;
    if (decay) {
        if (a.dlog == nullptr) return cudaErrorInvalidValue;
        decay_log2_prefix_kernel<<<(BH + 127) / 128, 128, 0, stream>>>(a.gamma, a.dlog, BH, nqt);
        dlog = a.dlog;
    }
    // The chunk start states (and the final state) first; the y kernel reads them.
    if (cc.nch > 1 || a.S != nullptr) {
        CUtensorMap sk_map, sv_map;
        if (!make_tmap_bf16_3d_swizzle(&sk_map, a.k, DF, a.N, BH, DF, CS, SL::K_SWIZZLE) ||
            !make_tmap_bf16_3d_swizzle(&sv_map, a.v, DV, a.N, BH, 64, CS, 128))
            return cudaErrorInvalidValue;
        auto sk = decay ? la_prefix_kernel<DF, DV, true> : la_prefix_kernel<DF, DV, false>;
        cudaError_t e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SL::SMEM_BYTES);
        if (e != cudaSuccess) return e;
        sk<<<BH * SL::NFT, kStateThreads, SL::SMEM_BYTES, stream>>>(sk_map, sv_map, a.S, a.z, spre, zpre, a.N,
                                                                     cc.R * (C / CS), cc.nch, a.packed ? 1 : 0,
                                                                     dlog, a.status, a.debug);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    using QL = QuadLayout<DF, DV>;
    CUtensorMap mq, mk, mv, mp;
    if (!make_tmap_bf16_3d_swizzle(&mq, a.q, DF, a.N, BH, DF, C, QL::QK_SWIZZLE) ||
        !make_tmap_bf16_3d_swizzle(&mk, a.k, DF, a.N, BH, DF, C, QL::QK_SWIZZLE) ||
        !make_tmap_bf16_3d_swizzle(&mv, a.v, DV, a.N, BH, 64, C, 128))
        return cudaErrorInvalidValue;
    // The state tiles: [BH * (nch-1)][NFT * 128 features][DV], loaded like V tiles.
    if (cc.nch > 1) {
        if (!make_tmap_bf16_3d_swizzle(&mp, spre, DV, (uint64_t)QL::NFT * 128, (uint64_t)BH * (cc.nch - 1), 64, C, 128))
            return cudaErrorInvalidValue;
    } else {
        mp = mv;                                         // never read: no virtual steps
    }
    auto qk = decay ? la_quad_kernel<DF, DV, true> : la_quad_kernel<DF, DV, false>;
    cudaError_t e = cudaFuncSetAttribute(qk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QL::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<long long>(nunits, num_sms);
    qk<<<grid, kQuadThreads, QL::SMEM_BYTES, stream>>>(mq, mk, mv, mp, static_cast<bf*>(a.y), a.N, BH, nqt, cc.R,
                                                       cc.nch, dlog, zpre, a.status, a.debug);
    return cudaGetLastError();
}

}  // namespace

bool la_prefill_quad_supported(int d_feat, int d_v) {
    return (d_feat == 16 || d_feat == 32) && (d_v == 64 || d_v == 128);
}

bool la_prefill_quad_chunk_ok(int chunk) { return chunk >= C && chunk % C == 0; }

size_t la_prefill_quad_workspace(int B, int H, int N, int d_feat, int d_v, int chunk) {
    if (!la_prefill_quad_supported(d_feat, d_v) || (chunk != 0 && !la_prefill_quad_chunk_ok(chunk))) return 0;
    const ChunkCfg cc = chunk_cfg(B, H, N, d_feat, d_v, chunk);
    return cc.s_bytes + cc.z_bytes;
}

cudaError_t launch_la_prefill_quad(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    if (!a.bf16 || !la_prefill_quad_supported(a.d_feat, a.d_v)) return cudaErrorInvalidValue;
    if (a.chunk != 0 && !la_prefill_quad_chunk_ok(a.chunk)) return cudaErrorInvalidValue;
    if (a.d_feat == 16 && a.d_v == 64) return launch_quad_typed<16, 64>(a, num_sms, stream);
    if (a.d_feat == 16 && a.d_v == 128) return launch_quad_typed<16, 128>(a, num_sms, stream);
    if (a.d_feat == 32 && a.d_v == 64) return launch_quad_typed<32, 64>(a, num_sms, stream);
    return launch_quad_typed<32, 128>(a, num_sms, stream);
}

}  // namespace based

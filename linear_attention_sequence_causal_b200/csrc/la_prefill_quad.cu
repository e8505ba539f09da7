// Tensor-core prefill of causal Taylor linear attention in its quadratic form,
// for the shapes whose state does not fit one SM's tensor memory (d' = 32, or
// dv = 128): y_i = sum_{j<=i} a_ij v_j / sum_{j<=i} a_ij, a_ij = 1 + s + s^2/2,
// s = q_i.k_j.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), App. B "Forward / Generation Prefill" computes each tile as
// a quadratic on-diagonal part plus a linear part read from the state of earlier
// tiles. At d' = 32 and dv = 128 the folded state [S | z] is 561 x 129 fp32
// (290 KB), more than the 256 KB of tensor memory of one SM. The quadratic form
// of the same sum is exact (every tile of the off-diagonal part is evaluated
// directly), needs no state during the sweep, and is a dense contraction:
//   S   = Q_qt K_kt^T                M=128 N=128 K=d'   -> TMEM
//   A   = 1 + S + S^2/2 (causal mask on the diagonal tile), bf16 over S in TMEM;
//         the row sums l of A accumulate in registers (fp32)
//   O  += A V_kt                     M=128 N=dv  K=128  (A operand in TMEM)
//   y   = O / l
// The final state S = phi(K)^T V, z = phi(K)^T 1 is a separate contraction over
// all tokens (la_state_kernel below).
//
// la_quad_kernel is persistent: one CTA per SM takes units (query tile qt, head
// bh) longest first (qt descending), and for each unit sweeps key tiles
// kt = 0..qt ("steps", numbered across the CTA's units). Roles (384 threads):
//   warp 0      lane 0: TMA loads of the unit's Q tile and each step's K and V
//               tiles into a 4-stage ring (rows past the sequence end read as 0);
//   warp 1      allocates TMEM; lane 0 issues S of every step, into S buffer
//               (step parity);
//   warps 2, 3  lane 0: O_g += P V of the steps of parity g, into accumulator
//               O_g (two issuers keep the tensor pipe busy: one thread alone
//               issues an MMA about every 117 cycles, while an M=128 N=128
//               K=16 product takes 64);
//   warps 4-7   A of the even steps (thread = query row = TMEM lane), and at
//               the end of a unit y = (O_0 + O_1) / l for columns [0, dv/2);
//   warps 8-11  the same for the odd steps and columns [dv/2, dv).
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

template <int DF, int DV>
struct QuadLayout {
    // Q and K tiles: K-major rows of d' bf16 (32 or 64 bytes) under the swizzle
    // of that width, 8-row atoms. V tile: MN-major under the 128-byte swizzle,
    // one 128-key x 64-value block per 64 values.
    static constexpr int QK_SWIZZLE = DF * 2;
    static constexpr uint32_t QK_BYTES = C * DF * 2;
    static constexpr uint32_t QK_SBO = 8 * DF * 2;
    static constexpr uint32_t V_BLOCK = C * 128;                          // 64 values x 128 keys
    static constexpr uint32_t V_BYTES = C * DV * 2;
    static constexpr uint32_t OFF_V = 0;                                   // [kStages]
    static constexpr uint32_t OFF_K = OFF_V + kStages * V_BYTES;          // [kStages]
    static constexpr uint32_t OFF_Q = OFF_K + kStages * QK_BYTES;         // [2] by unit parity
    static constexpr uint32_t OFF_L = OFF_Q + 2 * QK_BYTES;               // [kBufs][128] float row sums
    static constexpr uint32_t OFF_BAR = OFF_L + kBufs * C * 4;
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
};

enum {
    QB_FULL0, QB_FULL1, QB_FULL2, QB_FULL3,     // TMA: stage s (and the unit's Q) landed
    QB_EMPTY0, QB_EMPTY1, QB_EMPTY2, QB_EMPTY3, // O issuer commit: stage s read
    QB_SF0, QB_SF1, QB_SF2,                     // S issuer commit: S of buffer b ready
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
    const float* dlog;                          // decay: [BH][nqt] log2 prefix of gamma, or nullptr
};

__device__ __forceinline__ bool qwait(const QuadCtx& cx, int bar, uint32_t parity) {
    return mbar_wait(&cx.bars[bar], parity, cx.abort_flag, cx.status);
}

__device__ __forceinline__ void unit_of(const QuadCtx& cx, int u, int& qt, int& bh) {
    qt = cx.nqt - 1 - u / cx.BH;      // longest units first
    bh = u % cx.BH;
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
                                              const CUtensorMap* tv) {
    using L = QuadLayout<DF, DV>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int qt, bh;
        unit_of(cx, u, qt, bh);
        for (int kt = 0; kt <= qt; ++kt, ++step) {
            const int s = step % kStages;
            if (step >= kStages && !qwait(cx, QB_EMPTY0 + s, ((step / kStages) - 1) & 1)) { quad_drain(cx, last, lastp); return; }
            uint64_t* full = &cx.bars[QB_FULL0 + s];
            const int p = k_unit & 1;
            if (kt == 0) {
                // The unit's Q tile goes to the buffer of its parity once the S MMAs
                // of the unit two back are done with it; it lands with this stage.
                if (k_unit >= 2 && !qwait(cx, QB_QE0 + p, ((k_unit >> 1) - 1) & 1)) { quad_drain(cx, last, lastp); return; }
                mbar_expect_tx(full, L::QK_BYTES + L::QK_BYTES + L::V_BYTES);
                tma_load_3d(cx.sbase + L::OFF_Q + p * L::QK_BYTES, tq, full, 0, qt * C, bh);
            } else {
                mbar_expect_tx(full, L::QK_BYTES + L::V_BYTES);
            }
            tma_load_3d(cx.sbase + L::OFF_K + s * L::QK_BYTES, tk, full, 0, kt * C, bh);
#pragma unroll
            for (int h = 0; h < DV / 64; ++h)
                tma_load_3d(cx.sbase + L::OFF_V + s * L::V_BYTES + h * L::V_BLOCK, tv, full, 64 * h, kt * C, bh);
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

// ------------------------------------------------------------------ A warps (4-15)
// Group g (of kBufs) forms A for the steps with step % kBufs == g, in S / P
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
        const int step0 = step;
        float l0 = 0.0f, l1 = 0.0f;
        for (int kt = 0; kt <= qt; ++kt, ++step) {
            if (step % kBufs != g) continue;
            if (!qwait(cx, QB_SF0 + g, (step / kBufs) & 1)) return;
            tc_fence_after();
            const bool diag = kt == qt;          // keys j > i of the diagonal tile are masked
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
        const int nsteps = qt + 1;
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
            if (tok < cx.N) {
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
// S = Q K^T of every step (warp 1, lane 0), into S buffer step % kBufs.
template <int DF, int DV>
__device__ __forceinline__ void quad_s_issuer(const QuadCtx& cx, uint32_t tmem) {
    using L = QuadLayout<DF, DV>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int qt, bh;
        unit_of(cx, u, qt, bh);
        const int p = k_unit & 1;
        const uint64_t dq = smem_desc_swizzled(cx.sbase + L::OFF_Q + p * L::QK_BYTES, 16, L::QK_SBO, L::QK_SWIZZLE);
        for (int kt = 0; kt <= qt; ++kt, ++step) {
            const int s = step % kStages, b = step % kBufs;
            if (!qwait(cx, QB_FULL0 + s, (step / kStages) & 1)) { quad_drain(cx, last, lastp); return; }
            if (step >= kBufs && !qwait(cx, QB_OB0 + b, ((step / kBufs) - 1) & 1)) { quad_drain(cx, last, lastp); return; }
            tc_fence_after();
            const uint64_t dk = smem_desc_swizzled(cx.sbase + L::OFF_K + s * L::QK_BYTES, 16, L::QK_SBO, L::QK_SWIZZLE);
#pragma unroll
            for (int j = 0; j < DF / 16; ++j)       // K step of 16 = 32 bytes along the swizzled row
                mma_bf16(tmem + L::COL_S + b * C, dq + 2 * j, dk + 2 * j, L::ID_S, j > 0);
            mma_commit(&cx.bars[QB_SF0 + b]);
            last = &cx.bars[QB_SF0 + b];
            lastp = (step / kBufs) & 1;
            if (kt == qt) mma_commit(&cx.bars[QB_QE0 + p]);
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
        // O is free once every A thread has read out the previous unit.
        if (k_unit >= 1 && !qwait(cx, QB_OE, (k_unit - 1) & 1)) { quad_drain(cx, last, lastp); return; }
        bool first = true;
        for (int kt = 0; kt <= qt; ++kt, ++step) {
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
            for (int j = 0; j < C / 16; ++j)         // K step of 16 keys = 2048 bytes
                mma_bf16_ts(d_tmem, a_tmem + 8 * j, dv + ((j * 2048) >> 4), L::ID_O, (!first || j > 0) ? 1u : 0u);
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
               const __grid_constant__ CUtensorMap tv, __nv_bfloat16* __restrict__ y, int N, int BH, int nqt,
               const float* __restrict__ dlog, unsigned* status, unsigned debug) {
    using L = QuadLayout<DF, DV>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + 8 * QB_NUM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BAR + 8 * QB_NUM + 4);
    const QuadCtx cx{sbase, bars, reinterpret_cast<float*>(smem + L::OFF_L), abort_flag, status, N, BH, nqt,
                     nqt * BH, dlog};
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
        if (lane == 0) quad_producer<DF, DV>(cx, &tq, &tk, &tv);
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

// ------------------------------------------------------------------ final state
// S = phi(K)^T V and z = phi(K)^T 1 over all N tokens of a head, one CTA per
// (b, h, tile of 128 folded features), two CTAs per SM: D (TMEM lane = feature)
// += phi(K)^T [V | 1] per chunk of 64 tokens, M=128 N=dv+16 K=64. Warp 5 (lane
// 0) loads each chunk's K and V by TMA into a 2-stage ring; warps 0-3 (thread
// = token t, half fh of the tile's features) read k_t from shared memory and
// write their 64 features of phi(k_t); warp 4 allocates TMEM and issues the
// MMAs. The ones column of [V | 1] is a constant block of every stage. At the
// end warps 0-3 (thread = feature) write the feature's rows of the
// 1 + d' + d'^2 layout: the constant, the d' linear rows, and each folded pair
// x_a x_b as rows (a, b) and (b, a), each times 1/sqrt2 (the diagonal x_a^2
// carries its 1/sqrt2 already).
constexpr int kStateThreads = 192;
constexpr int CS = 64;               // tokens per chunk

// Folded feature f of [1, x_a, x_a x_b (a <= b, a-major)] as x[a] * x[b] * coef,
// x[DF] standing for the constant; coef 0 past the last feature.
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

// phi(k) of one token for 64 consecutive features from F0, from x (the token's
// k in fp32, x[DF] the constant). The feature pairs are evaluated at compile
// time (template arguments), so x stays in registers.
template <int DF, int F>
__device__ __forceinline__ float phi_elem(const float* x) {
    constexpr FeatPair fp = feat_pair(DF, F);
    return (x[fp.a] * x[fp.b]) * fp.coef;
}

template <int DF, int F0, int... E>
__device__ __forceinline__ uint4 phi_piece(const float* x, float u, std::integer_sequence<int, E...>) {
    const float f8[8] = {(phi_elem<DF, F0 + E>(x) * u)...};
    return pack_bf16x8(f8);
}

template <int DF, int F0, int... J>
__device__ __forceinline__ void state_phi_half_impl(const float* x, float u, uint32_t row, uint32_t sbo,
                                                    std::integer_sequence<int, J...>) {
    ((st_shared_v4(row + J * sbo, phi_piece<DF, F0 + 8 * J>(x, u, std::make_integer_sequence<int, 8>{}))), ...);
}

// Features [64 H, 64 H + 64) for the selector sel == H (H < HMAX).
template <int DF, int H, int HMAX>
__device__ __forceinline__ void state_phi_half(int sel, const float* x, float u, uint32_t row, uint32_t sbo) {
    if constexpr (H < HMAX) {
        if (sel == H) {
            state_phi_half_impl<DF, 64 * H>(x, u, row, sbo, std::make_integer_sequence<int, 8>{});
            return;
        }
        state_phi_half<DF, H + 1, HMAX>(sel, x, u, row, sbo);
    }
}

template <int DF, int DV>
struct StateLayout {
    static constexpr int DS = sym_feature_dim(DF);
    static constexpr int NFT = (DS + 127) / 128;
    static constexpr int NV = DV + 16;                   // [V | 1 | 0 ...]
    static constexpr uint32_t A_BYTES = 128 * CS * 2;    // phi(K)^T: M = feature, K = token, MN-major
    static constexpr uint32_t A_LBO = (128 / 8) * 128, A_SBO = 128;
    static constexpr int K_SWIZZLE = DF * 2;             // K tile: rows of d' bf16, swizzled
    static constexpr uint32_t K_BYTES = CS * DF * 2;
    static constexpr uint32_t V_BLOCK = CS * 128;        // 64 values x 64 tokens, 128-byte swizzle
    static constexpr uint32_t V_BYTES = (DV / 64 + 1) * V_BLOCK;   // the last block holds the ones column
    static constexpr uint32_t OFF_A = 0;                 // [2]
    static constexpr uint32_t OFF_V = 2 * A_BYTES;       // [2]
    static constexpr uint32_t OFF_K = OFF_V + 2 * V_BYTES;   // [2]
    static constexpr uint32_t OFF_F = OFF_K + 2 * K_BYTES;   // feature table: ia, ib (bytes), coef (float)
    static constexpr uint32_t OFF_BAR = OFF_F + 128 * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 128 + 1024;   // + alignment slack
    static_assert(2 * SMEM_BYTES <= 228 * 1024, "two CTAs per SM");
    static_assert(OFF_K % 1024 == 0 && K_BYTES % 1024 == 0, "tile alignment");
    static_assert(NFT <= 5, "feature tiles dispatched in la_state_kernel");
    static constexpr uint32_t TMEM_COLS = NV <= 128 ? 128 : 256;
    static constexpr uint32_t ID = idesc_bf16_f32(128, NV, true, true);
};

enum { SB_FULL0, SB_FULL1, SB_PHI0, SB_PHI1, SB_FREE0, SB_FREE1, SB_DONE, SB_NUM };

template <int DF, int DV, bool DECAY>
__global__ void __launch_bounds__(kStateThreads, 2)
la_state_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                float* __restrict__ S, float* __restrict__ z, int N, int packed, const float* __restrict__ dlog,
                unsigned* status, unsigned debug) {
    using L = StateLayout<DF, DV>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + 8 * SB_NUM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BAR + 8 * SB_NUM + 4);
    unsigned char* ftab = smem + L::OFF_F;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int bh = blockIdx.x / L::NFT;
    const int ft = blockIdx.x % L::NFT;
    const int f0 = ft * 128;
    const int nchunks = (N + CS - 1) / CS;
    const int nqt = (N + 127) / 128;                      // 128-token decay tiles

    if (tid < 128) {
        // Feature f0 + tid of the folded order [1, x_a, x_a x_b (a <= b, a-major)]
        // as x[ia] * x[ib] * coef, with x[DF] the constant (1, or 0 past the end).
        const int f = f0 + tid;
        int ia = DF, ib = DF;
        float coef = f < L::DS ? 1.0f : 0.0f;
        if (f >= 1 && f <= DF) {
            ia = f - 1;
        } else if (f > DF && f < L::DS) {
            int p = f - 1 - DF, a = 0;
            while (p >= DF - a) { p -= DF - a; ++a; }
            ia = a;
            ib = a + p;
            if (ia == ib) coef = kSqrtHalf;
        }
        ftab[8 * tid] = (unsigned char)ia;
        ftab[8 * tid + 1] = (unsigned char)ib;
        *reinterpret_cast<float*>(ftab + 8 * tid + 4) = coef;
    }
    // The ones block of both stages: value column 0 of every token row is 1, the
    // rest 0, stored under the 128-byte swizzle (logical piece 0 of row r sits
    // at physical piece r mod 8).
    for (int idx = tid; idx < 2 * CS * 8; idx += kStateThreads) {
        const int b = idx / (CS * 8), r = (idx / 8) % CS, c = idx % 8;
        const uint32_t at = sbase + L::OFF_V + b * L::V_BYTES + (DV / 64) * L::V_BLOCK + r * 128 + c * 16;
        st_shared_v4(at, make_uint4(c == (r & 7) ? 0x3F80u : 0u, 0u, 0u, 0u));
    }
    fence_proxy_async_smem();
    if (tid == 0) {
        for (int b = 0; b < SB_NUM; ++b) mbar_init(&bars[b], (b == SB_PHI0 || b == SB_PHI1) ? 128 : 1);
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
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (!mbar_wait(&bars[SB_FULL0 + b], (c >> 1) & 1, abort_flag, status)) break;
            // k of token t from the swizzled K tile (rows past N read as 0).
            float x[DF + 1];
            const uint32_t krow = sbase + L::OFF_K + b * L::K_BYTES;
#pragma unroll
            for (int j = 0; j < DF / 8; ++j) {
                const uint32_t o = t * (DF * 2) + 16 * j;
                const uint32_t phys = o ^ (((o >> 7) & (L::K_SWIZZLE / 16 - 1)) << 4);
                const uint4 u = ld_shared_v4(krow + phys);
                const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * j + 2 * e] = __uint_as_float(wd[e] << 16);
                    x[8 * j + 2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u);
                }
            }
            x[DF] = c * CS + t < N ? 1.0f : 0.0f;
            // Coarse decay: token t's contribution to the final state is scaled by the
            // product of gamma over the 128-token tiles after its own.
            const int tok = c * CS + t;
            const float u = DECAY ? exp2f(dlog[(size_t)bh * nqt + nqt - 1] - dlog[(size_t)bh * nqt + tok / 128]) : 1.0f;
            state_phi_half<DF, 0, 2 * L::NFT>(2 * ft + fh, x, u, arow + b * L::A_BYTES, L::A_SBO);
            fence_proxy_async_smem();
            mbar_arrive(&bars[SB_PHI0 + b]);
        }
    } else if (warp == 4) {
        if (lane == 0 && !(debug & DEBUG_SKIP_MMA)) {
            uint64_t* last = nullptr;
            uint32_t lastp = 0;
            for (int c = 0; c < nchunks; ++c) {
                const int b = c & 1;
                if (!mbar_wait(&bars[SB_PHI0 + b], (c >> 1) & 1, abort_flag, status)) break;
                tc_fence_after();
                const uint64_t da = smem_desc(sbase + L::OFF_A + b * L::A_BYTES, L::A_LBO, L::A_SBO);
                const uint64_t dv = smem_desc_sw128(sbase + L::OFF_V + b * L::V_BYTES, L::V_BLOCK, 1024);
#pragma unroll
                for (int j = 0; j < CS / 16; ++j)
                    mma_bf16(tmem, da + ((j * 2 * L::A_LBO) >> 4), dv + ((j * 2048) >> 4), L::ID,
                             (c > 0 || j > 0) ? 1u : 0u);
                mma_commit(&bars[SB_FREE0 + b]);
                last = &bars[SB_FREE0 + b];
                lastp = (c >> 1) & 1;
            }
            if (!*abort_flag) {
                mma_commit(&bars[SB_DONE]);
            } else if (last != nullptr) {
                const uint64_t t0 = global_ns();
                while (!mbar_try_wait(last, lastp) && global_ns() - t0 < kWaitLimitNs) {}
            }
        }
    } else if (lane == 0) {
        // TMA: chunk c into stage c mod 2 once the MMAs of chunk c - 2 are done with it.
        uint64_t* last = nullptr;
        uint32_t lastp = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (c >= 2 && !mbar_wait(&bars[SB_FREE0 + b], ((c >> 1) - 1) & 1, abort_flag, status)) break;
            uint64_t* full = &bars[SB_FULL0 + b];
            mbar_expect_tx(full, L::K_BYTES + (DV / 64) * L::V_BLOCK);
            tma_load_3d(sbase + L::OFF_K + b * L::K_BYTES, &tk, full, 0, c * CS, bh);
#pragma unroll
            for (int h = 0; h < DV / 64; ++h)
                tma_load_3d(sbase + L::OFF_V + b * L::V_BYTES + h * L::V_BLOCK, &tv, full, 64 * h, c * CS, bh);
            last = full;
            lastp = (c >> 1) & 1;
        }
        if (*abort_flag && last != nullptr) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(last, lastp) && global_ns() - t0 < kWaitLimitNs) {}
        }
    }

    // Epilogue: thread = feature f0 + tid (TMEM lane), rows of the full or the symmetric layout.
    if (warp < 4 && mbar_wait(&bars[SB_DONE], 0, abort_flag, status)) {
        tc_fence_after();
        const int f = f0 + tid;
        const int ia = ftab[8 * tid], ib = ftab[8 * tid + 1];
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
        const uint32_t taddr = tmem + (static_cast<uint32_t>(warp * 32) << 16);
#pragma unroll 1
        for (int m = 0; m < L::NV / 16; ++m) {
            float r[16];
            tmem_ld16(taddr + 16 * m, r);
            tmem_ld_wait();
            if (f >= L::DS) continue;
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const int col = 16 * m + e;
                const float val = r[e] * coef;
                if (col < DV) {
                    S[(hb * D + r0) * DV + col] = val;
                    if (r1 >= 0) S[(hb * D + r1) * DV + col] = val;
                } else if (col == DV) {
                    z[hb * D + r0] = val;
                    if (r1 >= 0) z[hb * D + r1] = val;
                }
            }
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

template <int DF, int DV>
cudaError_t launch_quad_typed(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    const int BH = a.B * a.H;
    const int nqt = (a.N + C - 1) / C;
    const long long nunits = (long long)nqt * BH;
    if (nunits > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    using QL = QuadLayout<DF, DV>;
    CUtensorMap mq, mk, mv;
    if (!make_tmap_bf16_3d_swizzle(&mq, a.q, DF, a.N, BH, DF, C, QL::QK_SWIZZLE) ||
        !make_tmap_bf16_3d_swizzle(&mk, a.k, DF, a.N, BH, DF, C, QL::QK_SWIZZLE) ||
        !make_tmap_bf16_3d_swizzle(&mv, a.v, DV, a.N, BH, 64, C, 128))
        return cudaErrorInvalidValue;
    auto qk = a.gamma != nullptr ? la_quad_kernel<DF, DV, true> : la_quad_kernel<DF, DV, false>;
    cudaError_t e = cudaFuncSetAttribute(qk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)QL::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<long long>(nunits, num_sms);
    const float* dlog = nullptr;
    if (a.gamma != nullptr) {
        if (a.dlog == nullptr) return cudaErrorInvalidValue;
        decay_log2_prefix_kernel<<<(BH + 127) / 128, 128, 0, stream>>>(a.gamma, a.dlog, BH, nqt);
        dlog = a.dlog;
    }
    qk<<<grid, kQuadThreads, QL::SMEM_BYTES, stream>>>(mq, mk, mv, static_cast<bf*>(a.y), a.N, BH, nqt, dlog,
                                                       a.status, a.debug);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.S == nullptr) return e;
    using SL = StateLayout<DF, DV>;
    CUtensorMap sk_map, sv_map;
    if (!make_tmap_bf16_3d_swizzle(&sk_map, a.k, DF, a.N, BH, DF, CS, SL::K_SWIZZLE) ||
        !make_tmap_bf16_3d_swizzle(&sv_map, a.v, DV, a.N, BH, 64, CS, 128))
        return cudaErrorInvalidValue;
    auto sk = a.gamma != nullptr ? la_state_kernel<DF, DV, true> : la_state_kernel<DF, DV, false>;
    e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SL::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    sk<<<BH * SL::NFT, kStateThreads, SL::SMEM_BYTES, stream>>>(sk_map, sv_map, a.S, a.z, a.N, a.packed ? 1 : 0,
                                                                 dlog, a.status, a.debug);
    return cudaGetLastError();
}

}  // namespace

bool la_prefill_quad_supported(int d_feat, int d_v) {
    return (d_feat == 16 || d_feat == 32) && (d_v == 64 || d_v == 128);
}

cudaError_t launch_la_prefill_quad(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    if (!a.bf16 || !la_prefill_quad_supported(a.d_feat, a.d_v)) return cudaErrorInvalidValue;
    if (a.d_feat == 16 && a.d_v == 64) return launch_quad_typed<16, 64>(a, num_sms, stream);
    if (a.d_feat == 16 && a.d_v == 128) return launch_quad_typed<16, 128>(a, num_sms, stream);
    if (a.d_feat == 32 && a.d_v == 64) return launch_quad_typed<32, 64>(a, num_sms, stream);
    return launch_quad_typed<32, 128>(a, num_sms, stream);
}

}  // namespace based

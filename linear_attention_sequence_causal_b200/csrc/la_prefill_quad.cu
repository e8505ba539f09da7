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
//   S   = Q_qt K_kt^T                M=128 N=128 K=d'       -> TMEM
//   A   = 1 + S + S^2/2 (causal mask on the diagonal tile), bf16 over S in TMEM
//   [O|l] += A [V_kt|1]              M=128 N=dv+16 K=128   (A operand in TMEM)
//   y   = O / l
// The ones column appended to V gives the denominators l from the same MMA,
// summed over exactly the bf16 values of A the numerators use.
// The final state S = phi(K)^T V, z = phi(K)^T 1 is a separate contraction over
// all tokens (la_state_kernel below).
//
// la_quad_kernel is persistent: one CTA per SM takes units (query tile qt, head
// bh) longest first (qt descending), and for each unit sweeps key tiles
// kt = 0..qt. Roles (448 threads):
//   warps 0-3   producers: cp.async of the unit's Q tile and each step's K and V
//               tiles (thread = token row) into a 4-stage ring, completing on the
//               stage's mbarrier; rows past the sequence end are zero-filled;
//   warps 4-7   A of the even steps: S -> A -> bf16 P in TMEM (thread = query
//               row); at the end of every unit, y = O / l to global memory;
//   warps 8-11  A of the odd steps (each group has its own S / P buffer);
//   warp 12     allocates TMEM; lane 0 issues S of every step;
//   warp 13     lane 0 issues [O|l] += P [V|1] of every step.
// Every hand-off is an mbarrier; every wait is bounded.
#include <algorithm>
#include <utility>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace based {
namespace {

using namespace tc;

constexpr int C = 128;               // query and key tile
constexpr int kStages = 4;
constexpr int kQuadThreads = 448;

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int DF, int DV>
struct QuadLayout {
    // K-major no-swizzle Q and K tiles (8-row x 16-byte core matrices), and the
    // MN-major no-swizzle V tile (core matrix = 8 keys x 8 values).
    static constexpr int NV = DV + 16;                                     // [V | 1 | 0 ...]
    static constexpr uint32_t QK_BYTES = C * DF * 2;
    static constexpr uint32_t V_BYTES = C * NV * 2;
    static constexpr uint32_t QK_LBO = 128, QK_SBO = (DF / 8) * 128;
    static constexpr uint32_t V_LBO = (NV / 8) * 128, V_SBO = 128;
    static constexpr uint32_t OFF_Q = 0;                                   // [2] by unit parity
    static constexpr uint32_t OFF_K = OFF_Q + 2 * QK_BYTES;                // [kStages]
    static constexpr uint32_t OFF_V = OFF_K + kStages * QK_BYTES;          // [kStages]
    static constexpr uint32_t OFF_BAR = OFF_V + kStages * V_BYTES;
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 256;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    // TMEM: S / P buffers 0 and 1 (128 fp32 columns each), then [O | l] (dv + 16 columns).
    static constexpr uint32_t COL_S = 0, COL_O = 2 * C;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t ID_S = idesc_bf16_f32(128, C, false, false);
    static constexpr uint32_t ID_O = idesc_bf16_f32(128, NV, false, true);
};

enum {
    QB_FULL0, QB_FULL1, QB_FULL2, QB_FULL3,     // producers -> S issuer: stage s (and the unit's Q) landed
    QB_EMPTY0, QB_EMPTY1, QB_EMPTY2, QB_EMPTY3, // O issuer commit: stage s read
    QB_SF0, QB_SF1,                             // S issuer commit: S of buffer b ready
    QB_PF0, QB_PF1,                             // A warps -> O issuer: P of buffer b written
    QB_OB0, QB_OB1,                             // O issuer commit: P of buffer b consumed
    QB_OF,                                      // O issuer commit: a unit's O complete
    QB_OE,                                      // A warps -> O issuer: O read out
    QB_QE0, QB_QE1,                             // S issuer commit: Q buffer p no longer read
    QB_NUM
};

struct QuadCtx {
    uint32_t sbase;
    uint64_t* bars;
    volatile int* abort_flag;
    unsigned* status;
    int N, BH, nqt, nunits;
};

__device__ __forceinline__ bool qwait(const QuadCtx& cx, int bar, uint32_t parity) {
    return mbar_wait(&cx.bars[bar], parity, cx.abort_flag, cx.status);
}

__device__ __forceinline__ void unit_of(const QuadCtx& cx, int u, int& qt, int& bh) {
    qt = cx.nqt - 1 - u / cx.BH;      // longest units first
    bh = u % cx.BH;
}

// ------------------------------------------------------------------ producers (warps 0-3)
template <int DF, int DV>
__device__ __forceinline__ void quad_producers(const QuadCtx& cx, int t, const __nv_bfloat16* __restrict__ q,
                                               const __nv_bfloat16* __restrict__ k,
                                               const __nv_bfloat16* __restrict__ v) {
    using L = QuadLayout<DF, DV>;
    const uint32_t cm = (t & 7) * 16;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int qt, bh;
        unit_of(cx, u, qt, bh);
        const size_t row0 = (size_t)bh * cx.N;
        for (int kt = 0; kt <= qt; ++kt, ++step) {
            const int s = step % kStages;
            if (step >= kStages && !qwait(cx, QB_EMPTY0 + s, ((step / kStages) - 1) & 1)) return;
            if (kt == 0) {
                // The unit's Q tile, into the buffer of its parity once the S MMAs of
                // the unit two back are done with it.
                const int p = k_unit & 1;
                if (k_unit >= 2 && !qwait(cx, QB_QE0 + p, ((k_unit >> 1) - 1) & 1)) return;
                const int tok = qt * C + t;
                const bool ok = tok < cx.N;
                const __nv_bfloat16* src = q + (row0 + (ok ? tok : 0)) * DF;
                const uint32_t dst = cx.sbase + L::OFF_Q + p * L::QK_BYTES + cm + (t >> 3) * L::QK_SBO;
#pragma unroll
                for (int j = 0; j < DF / 8; ++j) cp_async16(dst + j * L::QK_LBO, src + 8 * j, ok ? 16u : 0u);
            }
            const int key = kt * C + t;
            const bool ok = key < cx.N;
            const __nv_bfloat16* ks = k + (row0 + (ok ? key : 0)) * DF;
            const __nv_bfloat16* vs = v + (row0 + (ok ? key : 0)) * DV;
            const uint32_t kd = cx.sbase + L::OFF_K + s * L::QK_BYTES + cm + (t >> 3) * L::QK_SBO;
            const uint32_t vd = cx.sbase + L::OFF_V + s * L::V_BYTES + cm + (t >> 3) * L::V_LBO;
#pragma unroll
            for (int j = 0; j < DF / 8; ++j) cp_async16(kd + j * L::QK_LBO, ks + 8 * j, ok ? 16u : 0u);
#pragma unroll
            for (int j = 0; j < DV / 8; ++j) cp_async16(vd + j * L::V_SBO, vs + 8 * j, ok ? 16u : 0u);
            cp_async_arrive(&cx.bars[QB_FULL0 + s]);
        }
    }
    // Copies still landing when the CTA ends would write freed shared memory.
    asm volatile("cp.async.wait_all;" ::: "memory");
}

// ------------------------------------------------------------------ A warps (4-11)
// Group g (warps 4-7: g = 0, warps 8-11: g = 1) forms A for the steps of parity
// g, in S / P buffer g. Thread = query row i of the tile = TMEM lane i (wq =
// lane quadrant). Group 0 also writes y = O / l at the end of every unit.
template <int DF, int DV>
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
        for (int kt = 0; kt <= qt; ++kt, ++step) {
            if ((step & 1) != g) continue;
            if (!qwait(cx, QB_SF0 + g, (step >> 1) & 1)) return;
            tc_fence_after();
            const bool diag = kt == qt;          // keys j > i of the diagonal tile are masked
            // Quarter r reads S columns 32r..32r+31 and writes P columns
            // 16r..16r+15, which overlay S columns already read.
#pragma unroll 1
            for (int r = 0; r < 4; ++r) {
                float sv[32];
                tmem_ld16(sb + 32 * r, sv);
                tmem_ld16(sb + 32 * r + 16, sv + 16);
                tmem_ld_wait();
                uint32_t pw[16];
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float x0 = sv[2 * m], x1 = sv[2 * m + 1];
                    uint32_t wd = pack_bf16x2(fmaf(x0, fmaf(0.5f, x0, 1.0f), 1.0f), fmaf(x1, fmaf(0.5f, x1, 1.0f), 1.0f));
                    if (diag) {
                        const int j0 = 32 * r + 2 * m;
                        wd &= (j0 <= i ? 0x0000FFFFu : 0u) | (j0 + 1 <= i ? 0xFFFF0000u : 0u);
                    }
                    pw[m] = wd;
                }
                tmem_st16(sb + 16 * r, pw);
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&cx.bars[QB_PF0 + g]);
        }
        if (g != 0) continue;
        // Epilogue (group 0): y = O / l for this unit's rows.
        if (!qwait(cx, QB_OF, k_unit & 1)) return;
        tc_fence_after();
        const uint32_t ob = tmem + lane_off + L::COL_O;
        float lsum[16];
        tmem_ld16(ob + DV, lsum);
        tmem_ld_wait();
        const float inv = 1.0f / lsum[0];      // l >= 1/2 for every real row
        const int tok = qt * C + i;
        uint4* yp = reinterpret_cast<uint4*>(y + ((size_t)bh * cx.N + (tok < cx.N ? tok : 0)) * DV);
#pragma unroll 1
        for (int h = 0; h < DV / 32; ++h) {
            float o[32];
            tmem_ld16(ob + 32 * h, o);
            tmem_ld16(ob + 32 * h + 16, o + 16);
            tmem_ld_wait();
            if (h == DV / 32 - 1) {
                tc_fence_before();
                mbar_arrive(&cx.bars[QB_OE]);      // O may be overwritten by the next unit
            }
            if (tok < cx.N) {
#pragma unroll
                for (int p8 = 0; p8 < 4; ++p8) {
                    float t8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) t8[e] = o[8 * p8 + e] * inv;
                    yp[4 * h + p8] = pack_bf16x8(t8);
                }
            }
        }
    }
}

// ------------------------------------------------------------------ issuers
__device__ __forceinline__ void quad_drain(const QuadCtx& cx, uint64_t* bar, uint32_t parity) {
    if (!*cx.abort_flag || bar == nullptr) return;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity) && global_ns() - t0 < kWaitLimitNs) {}
}

// S = Q K^T of every step (warp 8, lane 0).
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
        const uint64_t dq = smem_desc(cx.sbase + L::OFF_Q + p * L::QK_BYTES, L::QK_LBO, L::QK_SBO);
        for (int kt = 0; kt <= qt; ++kt, ++step) {
            const int s = step % kStages, b = step & 1;
            if (!qwait(cx, QB_FULL0 + s, (step / kStages) & 1)) { quad_drain(cx, last, lastp); return; }
            if (step >= 2 && !qwait(cx, QB_OB0 + b, ((step >> 1) - 1) & 1)) { quad_drain(cx, last, lastp); return; }
            fence_proxy_async_smem();            // cp.async writes -> tensor-core reads
            tc_fence_after();
            const uint64_t dk = smem_desc(cx.sbase + L::OFF_K + s * L::QK_BYTES, L::QK_LBO, L::QK_SBO);
#pragma unroll
            for (int j = 0; j < DF / 16; ++j)
                mma_bf16(tmem + L::COL_S + b * C, dq + ((j * 2 * L::QK_LBO) >> 4), dk + ((j * 2 * L::QK_LBO) >> 4),
                         L::ID_S, j > 0);
            mma_commit(&cx.bars[QB_SF0 + b]);
            last = &cx.bars[QB_SF0 + b];
            lastp = (step >> 1) & 1;
            if (kt == qt) mma_commit(&cx.bars[QB_QE0 + p]);
        }
    }
    quad_drain(cx, last, lastp);
}

// O += P V of every step (warp 9, lane 0).
template <int DF, int DV>
__device__ __forceinline__ void quad_o_issuer(const QuadCtx& cx, uint32_t tmem) {
    using L = QuadLayout<DF, DV>;
    uint64_t* last = nullptr;
    uint32_t lastp = 0;
    int step = 0, k_unit = 0;
    for (int u = blockIdx.x; u < cx.nunits; u += gridDim.x, ++k_unit) {
        int qt, bh;
        unit_of(cx, u, qt, bh);
        for (int kt = 0; kt <= qt; ++kt, ++step) {
            const int s = step % kStages, b = step & 1;
            if (!qwait(cx, QB_PF0 + b, (step >> 1) & 1)) { quad_drain(cx, last, lastp); return; }
            if (kt == 0 && k_unit >= 1 && !qwait(cx, QB_OE, (k_unit - 1) & 1)) { quad_drain(cx, last, lastp); return; }
            fence_proxy_async_smem();            // cp.async writes of V -> tensor-core reads
            tc_fence_after();
            const uint64_t dv = smem_desc(cx.sbase + L::OFF_V + s * L::V_BYTES, L::V_LBO, L::V_SBO);
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16_ts(tmem + L::COL_O, tmem + L::COL_S + b * C + 8 * j, dv + ((j * 2 * L::V_LBO) >> 4), L::ID_O,
                            (kt > 0 || j > 0) ? 1u : 0u);
            mma_commit(&cx.bars[QB_EMPTY0 + s]);     // S and O of this step have read the stage
            mma_commit(&cx.bars[QB_OB0 + b]);
            last = &cx.bars[QB_OB0 + b];
            lastp = (step >> 1) & 1;
            if (kt == qt) {
                mma_commit(&cx.bars[QB_OF]);
                last = &cx.bars[QB_OF];
                lastp = k_unit & 1;
            }
        }
    }
    quad_drain(cx, last, lastp);
}

template <int DF, int DV>
__global__ void __launch_bounds__(kQuadThreads, 1)
la_quad_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
               const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ y, int N, int BH, int nqt,
               unsigned* status, unsigned debug) {
    using L = QuadLayout<DF, DV>;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + 8 * QB_NUM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BAR + 8 * QB_NUM + 4);
    const QuadCtx cx{smem_u32(smem), bars, abort_flag, status, N, BH, nqt, nqt * BH};
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int b = 0; b < QB_NUM; ++b) {
            const bool group = b <= QB_FULL3 || b == QB_PF0 || b == QB_PF1 || b == QB_OE;
            mbar_init(&bars[b], group ? 128 : 1);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 12) tmem_alloc(tmem_slot, L::TMEM_COLS);
    // The ones column of [V | 1] (and the zero pad after it) never changes:
    // write it once into every stage; cp.async only ever writes the V part.
    if (tid < C) {
        const uint32_t cm = (tid & 7) * 16;
        for (int s = 0; s < kStages; ++s) {
            const uint32_t vd = smem_u32(smem) + L::OFF_V + s * L::V_BYTES + cm + (tid >> 3) * L::V_LBO;
            st_shared_v4(vd + (DV / 8) * L::V_SBO, make_uint4(0x3F80u, 0u, 0u, 0u));
            st_shared_v4(vd + (DV / 8 + 1) * L::V_SBO, make_uint4(0, 0, 0, 0));
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const bool skip_mma = (debug & DEBUG_SKIP_MMA) != 0;   // testing: issue nothing, every waiter times out

    if (warp < 4) {
        quad_producers<DF, DV>(cx, tid, q, k, v);
    } else if (warp < 12) {
        quad_rows<DF, DV>(cx, tmem, (warp - 4) >> 2, warp & 3, lane, y);
    } else if (warp == 12) {
        if (lane == 0 && !skip_mma) quad_s_issuer<DF, DV>(cx, tmem);
    } else {
        if (lane == 0 && !skip_mma) quad_o_issuer<DF, DV>(cx, tmem);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 12) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, L::TMEM_COLS);
    }
}

// ------------------------------------------------------------------ final state
// S = phi(K)^T V and z = phi(K)^T 1 over all N tokens of a head, one CTA per
// (b, h, tile of 128 folded features): D (TMEM lane = feature) += phi(K)^T [V|1]
// per chunk of 128 tokens, M=128 N=dv+16 K=128. Warps 0-3 (thread = token)
// build the chunk's phi(K) rows for the tile's features and [V | 1] in shared
// memory (double-buffered); warp 4 allocates TMEM and issues the MMAs. At the
// end warps 0-3 (thread = feature) write the feature's rows of the
// 1 + d' + d'^2 layout: the constant, the d' linear rows, and each folded pair
// x_a x_b as rows (a, b) and (b, a), each times 1/sqrt2 (the diagonal x_a^2
// carries its 1/sqrt2 already).
constexpr int kStateThreads = 160;

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

// phi(k) of one token for the 128 features of tile FT, from x (the token's k in
// fp32, x[DF] the constant). The feature pairs are evaluated at compile time
// (template arguments), so x stays in registers.
template <int DF, int F>
__device__ __forceinline__ float phi_elem(const float* x) {
    constexpr FeatPair fp = feat_pair(DF, F);
    return (x[fp.a] * x[fp.b]) * fp.coef;
}

template <int DF, int FT, int J, int... E>
__device__ __forceinline__ uint4 phi_piece(const float* x, std::integer_sequence<int, E...>) {
    const float f8[8] = {phi_elem<DF, FT * 128 + 8 * J + E>(x)...};
    return pack_bf16x8(f8);
}

template <int DF, int FT, int... J>
__device__ __forceinline__ void state_phi_tile_impl(const float* x, uint32_t row, uint32_t sbo,
                                                    std::integer_sequence<int, J...>) {
    ((st_shared_v4(row + J * sbo, phi_piece<DF, FT, J>(x, std::make_integer_sequence<int, 8>{}))), ...);
}

template <int DF, int FT>
__device__ __forceinline__ void state_phi_tile(const float* x, uint32_t row, uint32_t sbo) {
    state_phi_tile_impl<DF, FT>(x, row, sbo, std::make_integer_sequence<int, 16>{});
}

template <int DF, int DV>
struct StateLayout {
    static constexpr int DS = sym_feature_dim(DF);
    static constexpr int NFT = (DS + 127) / 128;
    static constexpr int NV = DV + 16;                  // [V | 1 | 0 ...]
    static constexpr uint32_t A_BYTES = C * 128 * 2;    // phi(K)^T: M = feature, K = token, MN-major
    static constexpr uint32_t B_BYTES = C * NV * 2;     // [V|1]:    K = token, N = column, MN-major
    static constexpr uint32_t A_LBO = (128 / 8) * 128, A_SBO = 128;
    static constexpr uint32_t B_LBO = (NV / 8) * 128, B_SBO = 128;
    static constexpr uint32_t OFF_A = 0;                // [2]
    static constexpr uint32_t OFF_B = 2 * A_BYTES;      // [2]
    static constexpr uint32_t OFF_F = OFF_B + 2 * B_BYTES;   // feature table: ia, ib (bytes), coef (float)
    static constexpr uint32_t OFF_BAR = OFF_F + 128 * 8;
    static constexpr uint32_t SMEM_BYTES = OFF_BAR + 64;
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
    static_assert(NFT <= 5, "feature tiles dispatched in la_state_kernel");
    static constexpr uint32_t TMEM_COLS = NV <= 128 ? 128 : 256;
    static constexpr uint32_t ID = idesc_bf16_f32(128, NV, true, true);
};

enum { SB_FULL0, SB_FULL1, SB_FREE0, SB_FREE1, SB_DONE, SB_NUM };

template <int DF, int DV>
__global__ void __launch_bounds__(kStateThreads, 1)
la_state_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, float* __restrict__ S,
                float* __restrict__ z, int N, unsigned* status, unsigned debug) {
    using L = StateLayout<DF, DV>;
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_BAR + 8 * SB_NUM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BAR + 8 * SB_NUM + 4);
    unsigned char* ftab = smem + L::OFF_F;
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const size_t bh = blockIdx.x / L::NFT;
    const int f0 = (blockIdx.x % L::NFT) * 128;
    const int nchunks = (N + C - 1) / C;

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
    if (tid == 0) {
        for (int b = 0; b < SB_NUM; ++b) mbar_init(&bars[b], (b == SB_FULL0 || b == SB_FULL1) ? 128 : 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 4) tmem_alloc(tmem_slot, L::TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        const int t = tid;
        const uint32_t cm = (t & 7) * 16;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (c >= 2 && !mbar_wait(&bars[SB_FREE0 + b], ((c >> 1) - 1) & 1, abort_flag, status)) break;
            const int tok = c * C + t;
            const bool ok = tok < N;
            const uint4* kp = reinterpret_cast<const uint4*>(k + (bh * N + (ok ? tok : 0)) * DF);
            const uint4* vp = reinterpret_cast<const uint4*>(v + (bh * N + (ok ? tok : 0)) * DV);
            float x[DF + 1];
#pragma unroll
            for (int j = 0; j < DF / 8; ++j) {
                const uint4 u = ok ? __ldg(kp + j) : make_uint4(0, 0, 0, 0);
                const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    x[8 * j + 2 * e] = __uint_as_float(wd[e] << 16);
                    x[8 * j + 2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u);
                }
            }
            x[DF] = ok ? 1.0f : 0.0f;
            // [V | 1]: a 16-byte piece is 8 columns of token t
            const uint32_t vb = sbase + L::OFF_B + b * L::B_BYTES + cm + (t >> 3) * L::B_LBO;
#pragma unroll
            for (int j = 0; j < DV / 8; ++j) st_shared_v4(vb + j * L::B_SBO, ok ? __ldg(vp + j) : make_uint4(0, 0, 0, 0));
            st_shared_v4(vb + (DV / 8) * L::B_SBO, make_uint4(ok ? 0x3F80u : 0u, 0u, 0u, 0u));
            st_shared_v4(vb + (DV / 8 + 1) * L::B_SBO, make_uint4(0, 0, 0, 0));
            // phi(K) for the tile's 128 features: a 16-byte piece is 8 features of token t
            const uint32_t ab = sbase + L::OFF_A + b * L::A_BYTES + cm + (t >> 3) * L::A_LBO;
            switch (blockIdx.x % L::NFT) {
                case 0: state_phi_tile<DF, 0>(x, ab, L::A_SBO); break;
                case 1: state_phi_tile<DF, 1>(x, ab, L::A_SBO); break;
                case 2: state_phi_tile<DF, 2>(x, ab, L::A_SBO); break;
                case 3: state_phi_tile<DF, 3>(x, ab, L::A_SBO); break;
                default: state_phi_tile<DF, 4>(x, ab, L::A_SBO); break;
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars[SB_FULL0 + b]);
        }
    } else if (lane == 0 && !(debug & DEBUG_SKIP_MMA)) {
        uint64_t* last = nullptr;
        uint32_t lastp = 0;
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            if (!mbar_wait(&bars[SB_FULL0 + b], (c >> 1) & 1, abort_flag, status)) break;
            tc_fence_after();
            const uint64_t da = smem_desc(sbase + L::OFF_A + b * L::A_BYTES, L::A_LBO, L::A_SBO);
            const uint64_t db = smem_desc(sbase + L::OFF_B + b * L::B_BYTES, L::B_LBO, L::B_SBO);
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16(tmem, da + ((j * 2 * L::A_LBO) >> 4), db + ((j * 2 * L::B_LBO) >> 4), L::ID,
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

    // Epilogue: thread = feature f0 + tid (TMEM lane), rows of the full layout.
    if (warp < 4 && mbar_wait(&bars[SB_DONE], 0, abort_flag, status)) {
        tc_fence_after();
        const int f = f0 + tid;
        const int ia = ftab[8 * tid], ib = ftab[8 * tid + 1];
        constexpr int D = feature_dim(DF);
        int r0 = 0, r1 = -1;
        float coef = 1.0f;
        if (f == 0) {
            r0 = 0;
        } else if (f <= DF) {
            r0 = f;
        } else {
            r0 = 1 + DF + ia * DF + ib;
            if (ia != ib) { r1 = 1 + DF + ib * DF + ia; coef = kSqrtHalf; }
        }
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
                    S[(bh * D + r0) * DV + col] = val;
                    if (r1 >= 0) S[(bh * D + r1) * DV + col] = val;
                } else if (col == DV) {
                    z[bh * D + r0] = val;
                    if (r1 >= 0) z[bh * D + r1] = val;
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

template <int DF, int DV>
cudaError_t launch_quad_typed(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    using bf = __nv_bfloat16;
    const int BH = a.B * a.H;
    const int nqt = (a.N + C - 1) / C;
    const long long nunits = (long long)nqt * BH;
    if (nunits > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    auto qk = la_quad_kernel<DF, DV>;
    cudaError_t e = cudaFuncSetAttribute(qk, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)QuadLayout<DF, DV>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int grid = (int)std::min<long long>(nunits, num_sms);
    qk<<<grid, kQuadThreads, QuadLayout<DF, DV>::SMEM_BYTES, stream>>>(
        static_cast<const bf*>(a.q), static_cast<const bf*>(a.k), static_cast<const bf*>(a.v), static_cast<bf*>(a.y),
        a.N, BH, nqt, a.status, a.debug);
    e = cudaGetLastError();
    if (e != cudaSuccess || a.S == nullptr) return e;
    auto sk = la_state_kernel<DF, DV>;
    e = cudaFuncSetAttribute(sk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StateLayout<DF, DV>::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    sk<<<BH * StateLayout<DF, DV>::NFT, kStateThreads, StateLayout<DF, DV>::SMEM_BYTES, stream>>>(
        static_cast<const bf*>(a.k), static_cast<const bf*>(a.v), a.S, a.z, a.N, a.status, a.debug);
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

// Tensor-core (tcgen05 / TMEM) chunked prefill of causal Taylor linear attention.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), App. B "Forward / Generation Prefill": the feature map and
// the causal dot product are computed together, tile by tile; a tile's output is
// a quadratic on-diagonal part under a local causal mask plus a linear
// off-diagonal part read from the cumulative state of earlier tiles. With the
// K-state normalisation (App. D.4), for a chunk of C = 128 tokens:
//
//   s    = Q_c K_c^T                                  (tcgen05, M=128 N=128 K=16)
//   A    = mask(1 + s + s^2/2)                        (CUDA cores, from TMEM)
//   Y    = A [V_c | 1]  +  phi(Q_c) [S | z]           (tcgen05, N = 64 + 16)
//   y_c  = Y[:, :64] / Y[:, 64]                       (epilogue)
//   dS   = phi(K_c)^T [V_c | 1]                       (tcgen05, two 128-row tiles)
//   [S | z] += dS                                     (fp32, in registers)
//
// The ones column appended to V makes every product carry its own
// denominator: A [V | 1] yields the row sums of A, phi(Q)[S | z] yields
// phi(q).z, and phi(K)^T [V | 1] yields the increment of z.
//
// phi is never written to HBM: each token's thread forms phi(q_t) and phi(k_t)
// in registers and stores them (bf16) straight into the shared-memory operand
// tiles. The order-2 block is folded by symmetry, (q.k)^2/2 =
// sum_a (q_a^2/sqrt2)(k_a^2/sqrt2) + sum_{a<b} (q_a q_b)(k_a k_b), giving
// 1 + 16 + 136 = 153 features (padded to 160) instead of 273; the final state
// is expanded back to the 273-row layout on the way out.
//
// CTA roles (288 threads, one CTA per (b, h), TMEM fully owned):
//   warps 0-3  token threads: thread t owns token t of the chunk (TMEM lane t):
//              loads q, k, v, builds the operand tiles, turns s into A and
//              finishes y.
//   warps 4-7  state threads: own the rows of dS (TMEM lanes), keep the running
//              fp32 state [S | z] in registers and publish it as the bf16 B
//              operand of the next chunk's inter-chunk product.
//   warp 8     allocates TMEM; lane 0 issues every MMA and commit.
// All hand-offs go through mbarriers whose waits are bounded.
//
// Shared-memory operands use the canonical no-swizzle layouts (8-row x 16-byte
// core matrices, each a contiguous 128-byte block); each thread writes whole
// 16-byte rows of core matrices, so eight consecutive threads fill one block.
#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace based {
namespace {

using namespace tc;

constexpr int DF = 16;           // feature dim d'
constexpr int DV = 64;           // value dim
constexpr int C = 128;           // tokens per chunk
constexpr int DS = 153;          // distinct (symmetric) features
constexpr int KF = 160;          // DS padded to the MMA K step
constexpr int NV = 80;           // [V | 1] padded to the MMA N step
constexpr int kThreads = 288;

// Shared memory map (bytes). The update's second 128-row tile of phi(K)^T reads
// feature rows 128..255 of which only 128..159 exist; the rows beyond alias the
// next region (their products land in TMEM lanes that are never read).
constexpr uint32_t OFF_PK = 0;                          // phi(K)^T: M=feature, K=token, MN-major
constexpr uint32_t OFF_PQ = OFF_PK + KF * C * 2;        // phi(Q):   M=token, K=feature, K-major
constexpr uint32_t OFF_A = OFF_PQ + C * KF * 2;         // A:        M=token i, K=token j, K-major
constexpr uint32_t OFF_VA = OFF_A + C * C * 2;          // [V|1]:    N=column, K=token, MN-major
constexpr uint32_t OFF_SB = OFF_VA + C * NV * 2;        // [S|z]:    N=column, K=feature, MN-major
constexpr uint32_t OFF_Q = OFF_SB + KF * NV * 2;        // Q:        M=token, K=d', K-major
constexpr uint32_t OFF_K = OFF_Q + C * DF * 2;          // K:        N=token, K=d', K-major
constexpr uint32_t OFF_S1 = OFF_K + C * DF * 2;         // fp32 state rows 128..159 (warp 4)
constexpr uint32_t OFF_BAR = OFF_S1 + 32 * NV * 4;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 128;
static_assert(OFF_PK + (2 * C / 8 - 1) * 128 + (C / 8 - 1) * (KF / 8) * 128 + 128 <= SMEM_BYTES,
              "second update tile must stay inside shared memory");

// Core-matrix strides (bytes) of each operand: {K direction, M/N direction}.
constexpr uint32_t PK_LBO = (KF / 8) * 128, PK_SBO = 128;
constexpr uint32_t PQ_LBO = 128, PQ_SBO = (KF / 8) * 128;
constexpr uint32_t A_LBO = 128, A_SBO = (C / 8) * 128;
constexpr uint32_t VA_LBO = (NV / 8) * 128, VA_SBO = 128;
constexpr uint32_t SB_LBO = (NV / 8) * 128, SB_SBO = 128;
constexpr uint32_t QK_LBO = 128, QK_SBO = (DF / 8) * 128;

// TMEM columns.
constexpr uint32_t COL_S = 0;      // s = Q K^T, 128 columns
constexpr uint32_t COL_Y = 128;    // Y, 80 columns
constexpr uint32_t COL_D0 = 256;   // dS rows 0..127, 80 columns
constexpr uint32_t COL_D1 = 384;   // dS rows 128..255, 80 columns
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_QK = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t ID_AV = idesc_bf16_f32(128, NV, false, true);
constexpr uint32_t ID_UPD = idesc_bf16_f32(128, NV, true, true);
constexpr uint32_t ID_INT = idesc_bf16_f32(128, NV, false, true);

enum { BAR_IN, BAR_S, BAR_A, BAR_Y, BAR_SB, NUM_BARS };

// Emit phi_sym(x) as 20 packed 16-byte pieces of 8 features, in feature order
// [1, x_0..x_15, x_a x_b (a <= b, a-major; x_a^2 carries 1/sqrt2), 0 x 7].
template <typename Store>
__device__ __forceinline__ void emit_phi(const float* x, Store store) {
    float buf[8];
    int n = 0, piece = 0;
    auto push = [&](float val) {
        buf[n++] = val;
        if (n == 8) {
            store(piece++, pack_bf16x8(buf));
            n = 0;
        }
    };
    push(1.0f);
#pragma unroll
    for (int a = 0; a < DF; ++a) push(x[a]);
#pragma unroll
    for (int a = 0; a < DF; ++a) {
#pragma unroll
        for (int b = a; b < DF; ++b) push(a == b ? (x[a] * x[a]) * kSqrtHalf : x[a] * x[b]);
    }
#pragma unroll
    for (int f = DS; f < KF; ++f) push(0.0f);
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float* x) {
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        x[2 * i] = __uint_as_float(w[i] << 16);
        x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// (a, b) of folded pair index p (a <= b, a-major).
__device__ __forceinline__ void pair_of(int p, int& a, int& b) {
    a = 0;
    while (p >= DF - a) { p -= DF - a; ++a; }
    b = a + p;
}

__global__ void __launch_bounds__(kThreads, 1)
la_prefill_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ y,
                     float* __restrict__ S, float* __restrict__ z, int N, unsigned* status) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_BAR + 8 * NUM_BARS + 4);
    const uint32_t sbase = smem_u32(smem);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const size_t bh = blockIdx.x;
    const int nchunks = (N + C - 1) / C;

    if (tid == 0) {
        mbar_init(&bars[BAR_IN], 128);
        mbar_init(&bars[BAR_S], 1);
        mbar_init(&bars[BAR_A], 128);
        mbar_init(&bars[BAR_Y], 1);
        mbar_init(&bars[BAR_SB], 128);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 8) tmem_alloc(tmem_base_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;

    if (warp < 4) {
        // ------------------------------------------------------------ token threads
        const int t = tid;                                   // token within chunk == TMEM lane
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const uint32_t cm = (t & 7) * 16;                    // row within a core matrix
        for (int c = 0; c < nchunks; ++c) {
            const int t0 = c * C;
            const int nv = min(C, N - t0);
            const bool valid = t < nv;
            const size_t row = bh * (size_t)N + t0 + t;
            uint4 qr[2], kr[2], vr[8];
            if (valid) {
                const uint4* qp = reinterpret_cast<const uint4*>(q + row * DF);
                const uint4* kp = reinterpret_cast<const uint4*>(k + row * DF);
                const uint4* vp = reinterpret_cast<const uint4*>(v + row * DV);
                qr[0] = __ldg(qp); qr[1] = __ldg(qp + 1);
                kr[0] = __ldg(kp); kr[1] = __ldg(kp + 1);
#pragma unroll
                for (int i = 0; i < 8; ++i) vr[i] = __ldg(vp + i);
            } else {
                qr[0] = qr[1] = kr[0] = kr[1] = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int i = 0; i < 8; ++i) vr[i] = make_uint4(0, 0, 0, 0);
            }
            // Q, K tiles (K-major, 2 core matrices along d')
            const uint32_t qk_off = cm + (t >> 3) * QK_SBO;
            st_shared_v4(sbase + OFF_Q + qk_off, qr[0]);
            st_shared_v4(sbase + OFF_Q + qk_off + QK_LBO, qr[1]);
            st_shared_v4(sbase + OFF_K + qk_off, kr[0]);
            st_shared_v4(sbase + OFF_K + qk_off + QK_LBO, kr[1]);
            // [V | 1] (MN-major: 16-byte piece = 8 columns of token t)
            const uint32_t va_off = OFF_VA + cm + (t >> 3) * VA_LBO;
#pragma unroll
            for (int i = 0; i < 8; ++i) st_shared_v4(sbase + va_off + i * VA_SBO, vr[i]);
            st_shared_v4(sbase + va_off + 8 * VA_SBO,
                         make_uint4(valid ? 0x3F80u : 0u, 0u, 0u, 0u));   // bf16 1.0 in column 64
            st_shared_v4(sbase + va_off + 9 * VA_SBO, make_uint4(0, 0, 0, 0));
            // phi(Q) (K-major rows) and phi(K)^T (MN-major columns); padded tokens get phi(k) = 0
            float xq[DF], xk[DF];
            unpack_bf16x8(qr[0], xq);
            unpack_bf16x8(qr[1], xq + 8);
            unpack_bf16x8(kr[0], xk);
            unpack_bf16x8(kr[1], xk + 8);
            const uint32_t pq_off = OFF_PQ + cm + (t >> 3) * PQ_SBO;
            emit_phi(xq, [&](int j, uint4 u) { st_shared_v4(sbase + pq_off + j * PQ_LBO, u); });
            const uint32_t pk_off = OFF_PK + cm + (t >> 3) * PK_LBO;
            if (valid) {
                emit_phi(xk, [&](int j, uint4 u) { st_shared_v4(sbase + pk_off + j * PK_SBO, u); });
            } else {
#pragma unroll
                for (int j = 0; j < KF / 8; ++j) st_shared_v4(sbase + pk_off + j * PK_SBO, make_uint4(0, 0, 0, 0));
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[BAR_IN]);

            // s -> A (rows of s live in this thread's TMEM lane)
            if (!mbar_wait(&bars[BAR_S], c & 1, abort_flag, status)) break;
            tc_fence_after();
            const uint32_t a_off = OFF_A + cm + (t >> 3) * A_SBO;
#pragma unroll
            for (int b = 0; b < C / 32; ++b) {
                if (b > warp) {                              // whole 32-column block above the diagonal
#pragma unroll
                    for (int j = 0; j < 4; ++j) st_shared_v4(sbase + a_off + (4 * b + j) * A_LBO, make_uint4(0, 0, 0, 0));
                    continue;
                }
                float s[32];
                tmem_ld16(lane_base + COL_S + 32 * b, s);
                tmem_ld16(lane_base + COL_S + 32 * b + 16, s + 16);
                tmem_ld_wait();
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float a8[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int col = 32 * b + 8 * j + e;
                        const float sv = s[8 * j + e];
                        a8[e] = col <= t ? fmaf(sv, fmaf(0.5f, sv, 1.0f), 1.0f) : 0.0f;
                    }
                    st_shared_v4(sbase + a_off + (4 * b + j) * A_LBO, pack_bf16x8(a8));
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[BAR_A]);

            // y = Y[:, :64] / Y[:, 64]
            if (!mbar_wait(&bars[BAR_Y], c & 1, abort_flag, status)) break;
            tc_fence_after();
            float yv[NV];
#pragma unroll
            for (int m = 0; m < NV / 16; ++m) tmem_ld16(lane_base + COL_Y + 16 * m, yv + 16 * m);
            tmem_ld_wait();
            if (valid) {
                const float inv = 1.0f / yv[DV];
                uint4* yp = reinterpret_cast<uint4*>(y + row * DV);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float o[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) o[e] = yv[8 * i + e] * inv;
                    yp[i] = pack_bf16x8(o);
                }
            }
            tc_fence_before();
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ state threads
        const int wq = warp - 4;
        const int f0 = wq * 32 + lane;                       // feature row of tile 0
        const bool has_tile1 = (wq == 0);                    // rows 128..159 live in lanes 0..31
        const int f1 = 128 + lane;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        float S0[NV];
#pragma unroll
        for (int i = 0; i < NV; ++i) S0[i] = 0.f;
        // Rows 128..159 (folded features 128..152 plus zero padding) are few: they
        // stay in shared memory, one 80-float row per lane of warp 4.
        float* S1 = reinterpret_cast<float*>(smem + OFF_S1) + lane * NV;
        if (has_tile1) {
            for (int i = 0; i < NV; ++i) S1[i] = 0.f;
        }
        for (int c = 0; c < nchunks; ++c) {
            if (!mbar_wait(&bars[BAR_Y], c & 1, abort_flag, status)) break;
            tc_fence_after();
#pragma unroll
            for (int m = 0; m < NV / 16; ++m) {
                float d[16];
                tmem_ld16(lane_base + COL_D0 + 16 * m, d);
                tmem_ld_wait();
#pragma unroll
                for (int i = 0; i < 16; ++i) S0[16 * m + i] += d[i];
            }
            if (has_tile1) {
#pragma unroll
                for (int m = 0; m < NV / 16; ++m) {
                    float d[16];
                    tmem_ld16(lane_base + COL_D1 + 16 * m, d);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i) S1[16 * m + i] += (f1 < DS) ? d[i] : 0.f;
                }
            }
            if (c + 1 < nchunks) {
                const uint32_t sb0 = sbase + OFF_SB + (f0 & 7) * 16 + (f0 >> 3) * SB_LBO;
#pragma unroll
                for (int j = 0; j < NV / 8; ++j) st_shared_v4(sb0 + j * SB_SBO, pack_bf16x8(S0 + 8 * j));
                if (has_tile1) {
                    const uint32_t sb1 = sbase + OFF_SB + (f1 & 7) * 16 + (f1 >> 3) * SB_LBO;
#pragma unroll
                    for (int j = 0; j < NV / 8; ++j) {
                        float t8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) t8[e] = S1[8 * j + e];
                        st_shared_v4(sb1 + j * SB_SBO, pack_bf16x8(t8));
                    }
                }
                fence_proxy_async_smem();
            }
            tc_fence_before();
            mbar_arrive(&bars[BAR_SB]);
        }
        if (S != nullptr && !*abort_flag) {
            // Expand the folded state to the 1 + d' + d'^2 row layout.
            auto write_rows = [&](const float* Sr, int f) {
                if (f >= DS) return;
                int rows[2], nrows = 1;
                float coef = 1.0f;
                if (f <= DF) {
                    rows[0] = f;
                } else {
                    int a, b;
                    pair_of(f - 1 - DF, a, b);
                    rows[0] = 1 + DF + a * DF + b;
                    if (a != b) { rows[1] = 1 + DF + b * DF + a; nrows = 2; coef = kSqrtHalf; }
                }
                for (int i = 0; i < nrows; ++i) {
                    float4* dst = reinterpret_cast<float4*>(S + (bh * feature_dim(DF) + rows[i]) * DV);
#pragma unroll
                    for (int j = 0; j < DV / 4; ++j)
                        dst[j] = make_float4(Sr[4 * j] * coef, Sr[4 * j + 1] * coef, Sr[4 * j + 2] * coef,
                                             Sr[4 * j + 3] * coef);
                    z[bh * feature_dim(DF) + rows[i]] = Sr[DV] * coef;
                }
            };
            write_rows(S0, f0);
            if (has_tile1) write_rows(S1, f1);
        }
    } else if (lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        const uint64_t dq = smem_desc(sbase + OFF_Q, QK_LBO, QK_SBO);
        const uint64_t dk = smem_desc(sbase + OFF_K, QK_LBO, QK_SBO);
        int issued = 0;
        for (int c = 0; c < nchunks; ++c) {
            if (!mbar_wait(&bars[BAR_IN], c & 1, abort_flag, status)) break;
            tc_fence_after();
            mma_bf16(tmem + COL_S, dq, dk, ID_QK, 0);
            mma_commit(&bars[BAR_S]);

            if (!mbar_wait(&bars[BAR_A], c & 1, abort_flag, status)) break;
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < C / 16; ++j)
                mma_bf16(tmem + COL_Y, smem_desc(sbase + OFF_A + j * 2 * A_LBO, A_LBO, A_SBO),
                         smem_desc(sbase + OFF_VA + j * 2 * VA_LBO, VA_LBO, VA_SBO), ID_AV, j > 0);
            if (c > 0) {                                     // state threads done with dS and [S|z] of c-1
                if (!mbar_wait(&bars[BAR_SB], (c - 1) & 1, abort_flag, status)) break;
                tc_fence_after();
            }
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int j = 0; j < C / 16; ++j)
                    mma_bf16(tmem + (r == 0 ? COL_D0 : COL_D1),
                             smem_desc(sbase + OFF_PK + r * 16 * PK_SBO + j * 2 * PK_LBO, PK_LBO, PK_SBO),
                             smem_desc(sbase + OFF_VA + j * 2 * VA_LBO, VA_LBO, VA_SBO), ID_UPD, j > 0);
            }
            if (c > 0) {
#pragma unroll
                for (int j = 0; j < KF / 16; ++j)
                    mma_bf16(tmem + COL_Y, smem_desc(sbase + OFF_PQ + j * 2 * PQ_LBO, PQ_LBO, PQ_SBO),
                             smem_desc(sbase + OFF_SB + j * 2 * SB_LBO, SB_LBO, SB_SBO), ID_INT, 1);
            }
            mma_commit(&bars[BAR_Y]);
            issued = c + 1;
        }
        // Never free TMEM under an MMA still in flight: wait (bounded) for the last commit.
        if (issued > 0 && *abort_flag) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(&bars[BAR_Y], (issued - 1) & 1) && global_ns() - t0 < kWaitLimitNs) {}
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 8) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace

bool la_prefill_tc_supported(int d_feat, int d_v, int chunk) {
    return d_feat == DF && d_v == DV && chunk == C;
}

size_t la_prefill_tc_workspace(int, int, int, int, int, int, int) { return 0; }

cudaError_t launch_la_prefill_tc(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    (void)num_sms;
    if (!la_prefill_tc_supported(a.d_feat, a.d_v, a.chunk) || !a.bf16) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(la_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    la_prefill_tc_kernel<<<a.B * a.H, kThreads, SMEM_BYTES, stream>>>(
        static_cast<const __nv_bfloat16*>(a.q), static_cast<const __nv_bfloat16*>(a.k),
        static_cast<const __nv_bfloat16*>(a.v), static_cast<__nv_bfloat16*>(a.y), a.S, a.z, a.N, a.status);
    return cudaGetLastError();
}

}  // namespace based

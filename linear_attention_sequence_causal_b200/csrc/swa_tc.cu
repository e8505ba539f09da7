// Tensor-core (tcgen05 / TMEM) sliding-window softmax attention prefill, bf16, head dim 64, w <= 64.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), §4 "Local Exact Attention": exact softmax over the w most
// recent keys (the query's own position included), O(Nw) work.
//
// One CTA computes 128 consecutive queries [i0, i0 + 128) of one head. Every key
// those queries can see lies in the 192-key span [i0 - 64, i0 + 128), so a whole
// tile needs exactly one score block and one value block -- no running softmax:
//   TMA    Q [128 x 64], K and V [192 x 64] (128-byte swizzle; rows before the
//          sequence start or past its end arrive as zeros)
//   MMA    S = Q K^T              M=128 N=192 K=64   -> TMEM (192 columns)
//   CUDA   row i keeps only its band i0+i-w < j <= i0+i; p = exp(scale*(s - max)),
//          written as bf16 P over the Q/K buffers, l = sum of the rounded p
//   MMA    O = P V                M=128 N=64 K=192   -> TMEM (64 columns)
//   CUDA   y = O / l  -> global
// A warp's 32 query rows touch only 96 of the 192 score columns; it reads just
// those from TMEM and writes zeros for the rest of its P rows.
//
// Roles: warps 0-3 own query rows (TMEM lanes); warp 4 allocates TMEM and its
// lane 0 issues the TMA loads, both MMAs and the commits, while lanes 1-31 copy
// the tile's share of the last w tokens into the ring KV cache (slot t mod w;
// the first tile also zeroes the slots a prompt shorter than w never fills).
// Waits are bounded.
#include <cuda.h>
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma_host.h"

namespace based {
namespace {

using namespace tc;

constexpr int QT = 128;              // queries per CTA
constexpr int KW = 192;              // keys per CTA: [i0 - 64, i0 + 128)
constexpr int HD = 64;               // head dim
constexpr int kThreads = 160;

// Shared memory (offsets from a 1024-aligned base). P (3 atom columns of
// 128 rows x 128 B) reuses Q, K and the pad after them once S is computed.
constexpr uint32_t OFF_Q = 0;                      // 16 KB
constexpr uint32_t OFF_K = OFF_Q + QT * HD * 2;    // 24 KB
constexpr uint32_t OFF_P = 0;                      // 48 KB, after S completes
constexpr uint32_t OFF_V = 3 * QT * 128;           // 24 KB
constexpr uint32_t OFF_BAR = OFF_V + KW * HD * 2;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 64 + 1024;   // + alignment slack
static_assert(OFF_K + KW * HD * 2 <= OFF_V, "P region must cover Q and K");
constexpr uint32_t TX_BYTES = QT * HD * 2 + 2 * KW * HD * 2;

constexpr uint32_t COL_S = 0;        // 192 columns
constexpr uint32_t COL_O = 192;      // 64 columns
constexpr uint32_t TMEM_COLS = 256;

constexpr uint32_t ID_S = idesc_bf16_f32(128, KW, false, false);
constexpr uint32_t ID_O = idesc_bf16_f32(128, HD, false, true);

enum { BAR_LOAD, BAR_S, BAR_P, BAR_O, NUM_BARS };

__global__ void __launch_bounds__(kThreads)
swa_prefill_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ y,
                      __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache, int N, int w,
                      float scale_log2, unsigned* status, unsigned debug) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_BAR + 8 * NUM_BARS + 4);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int i0 = blockIdx.x * QT;
    const int bh = blockIdx.y;
    const int kb = i0 - 64;            // first key of the span

    if (tid == 0) {
        mbar_init(&bars[BAR_LOAD], 1);
        mbar_init(&bars[BAR_S], 1);
        mbar_init(&bars[BAR_P], 128);
        mbar_init(&bars[BAR_O], 1);
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 4) tmem_alloc(tmem_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp < 4) {
        const int i = tid;                          // query row == TMEM lane
        const int qi = i0 + i;
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        float l = 1.0f;
        if (mbar_wait(&bars[BAR_S], 0, abort_flag, status)) {
            tc_fence_after();
            // Columns [32*warp, 32*warp + 96) hold every key of this warp's rows.
            float s[96];
#pragma unroll
            for (int m = 0; m < 6; ++m) tmem_ld16(lane_base + COL_S + 32 * warp + 16 * m, s + 16 * m);
            tmem_ld_wait();
            const int jl_lo = i + 65 - w;           // band in span coordinates, inclusive
            const int jl_hi = i + 64;
            float mx = -INFINITY;
#pragma unroll
            for (int c = 0; c < 96; ++c) {
                const int jl = 32 * warp + c;
                const bool ok = jl >= jl_lo && jl <= jl_hi && kb + jl >= 0 && qi < N;
                s[c] = ok ? s[c] * scale_log2 : -INFINITY;
                mx = fmaxf(mx, s[c]);
            }
            float sum = 0.f;
            // P row i: span chunks [4*warp, 4*warp + 12) carry the band, the rest are zero.
            const uint32_t prow = sbase + OFF_P;
#pragma unroll
            for (int c8 = 0; c8 < KW / 8; ++c8) {
                if (c8 < 4 * warp || c8 >= 4 * warp + 12)
                    st_shared_v4(prow + (c8 >> 3) * (QT * 128) + sw128_offset(i, c8 & 7), make_uint4(0, 0, 0, 0));
            }
#pragma unroll
            for (int cc = 0; cc < 12; ++cc) {
                const int c8 = 4 * warp + cc;
                float p[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float t = s[8 * cc + e];
                    p[e] = (t == -INFINITY) ? 0.f : exp2f(t - mx);
                }
                const uint4 u = pack_bf16x8(p);
                // normalise with the bf16 values the MMA will see
                const uint32_t wds[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    sum += __uint_as_float(wds[e] << 16) + __uint_as_float(wds[e] & 0xFFFF0000u);
                st_shared_v4(prow + (c8 >> 3) * (QT * 128) + sw128_offset(i, c8 & 7), u);
            }
            l = sum > 0.f ? sum : 1.0f;
            fence_proxy_async_smem();
            tc_fence_before();
            mbar_arrive(&bars[BAR_P]);
            if (mbar_wait(&bars[BAR_O], 0, abort_flag, status)) {
                tc_fence_after();
                float o[HD];
#pragma unroll
                for (int m = 0; m < HD / 16; ++m) tmem_ld16(lane_base + COL_O + 16 * m, o + 16 * m);
                tmem_ld_wait();
                if (qi < N) {
                    const float inv = 1.0f / l;
                    uint4* yp = reinterpret_cast<uint4*>(y + ((size_t)bh * N + qi) * HD);
#pragma unroll
                    for (int c8 = 0; c8 < HD / 8; ++c8) {
                        float t[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) t[e] = o[8 * c8 + e] * inv;
                        yp[c8] = pack_bf16x8(t);
                    }
                }
            }
        }
    } else if (lane == 0) {
        mbar_expect_tx(&bars[BAR_LOAD], TX_BYTES);
        tma_load_3d(sbase + OFF_Q, &tq, &bars[BAR_LOAD], 0, i0, bh);
        tma_load_3d(sbase + OFF_K, &tk, &bars[BAR_LOAD], 0, kb, bh);
        tma_load_3d(sbase + OFF_V, &tv, &bars[BAR_LOAD], 0, kb, bh);
        bool ok = mbar_wait(&bars[BAR_LOAD], 0, abort_flag, status);
        int committed = 0;
        if (debug & DEBUG_SKIP_MMA) ok = false;             // testing: leave every waiter to time out
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < HD / 16; ++j)
                mma_bf16(tmem + COL_S, smem_desc_sw128(sbase + OFF_Q + 32 * j, 16, 1024),
                         smem_desc_sw128(sbase + OFF_K + 32 * j, 16, 1024), ID_S, j > 0);
            mma_commit(&bars[BAR_S]);
            committed = 1;
            ok = mbar_wait(&bars[BAR_P], 0, abort_flag, status);
        }
        if (ok) {
            tc_fence_after();
#pragma unroll
            for (int j = 0; j < KW / 16; ++j)
                mma_bf16(tmem + COL_O,
                         smem_desc_sw128(sbase + OFF_P + (j >> 2) * (QT * 128) + 32 * (j & 3), 16, 1024),
                         smem_desc_sw128(sbase + OFF_V + j * 2048, 16, 1024), ID_O, j > 0);
            mma_commit(&bars[BAR_O]);
            committed = 2;
        }
        // Never free TMEM under an MMA still in flight.
        if (*abort_flag && committed > 0) {
            const uint64_t t0 = global_ns();
            uint64_t* last = committed == 2 ? &bars[BAR_O] : &bars[BAR_S];
            while (!mbar_try_wait(last, 0) && global_ns() - t0 < kWaitLimitNs) {}
        }
        // The TMA load may still be landing if its wait gave up: wait (bounded) for it too.
        if (!ok && committed == 0) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(&bars[BAR_LOAD], 0) && global_ns() - t0 < kWaitLimitNs) {}
        }
    }

    else if (k_cache != nullptr) {
        // Ring cache: tokens u in [max(i0, N - w), min(i0 + QT, N)) go to slot u mod w.
        const int u0 = max(i0, N - w), u1 = min(i0 + QT, N);
        const size_t head = (size_t)bh * N;
        const size_t ring = (size_t)bh * w;
        for (int e = lane - 1; e < (u1 - u0) * 16; e += 31) {
            const int u = u0 + (e >> 4), c = e & 15;
            const uint4* src = reinterpret_cast<const uint4*>((c < 8 ? k : v) + (head + u) * HD) + (c & 7);
            uint4* dst = reinterpret_cast<uint4*>((c < 8 ? k_cache : v_cache) + (ring + u % w) * HD) + (c & 7);
            *dst = __ldg(src);
        }
        if (blockIdx.x == 0) {
            for (int e = lane - 1; e < max(0, w - N) * 16; e += 31) {
                const int slot = N + (e >> 4), c = e & 15;
                uint4* dst = reinterpret_cast<uint4*>((c < 8 ? k_cache : v_cache) + (ring + slot) * HD) + (c & 7);
                *dst = make_uint4(0, 0, 0, 0);
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 4) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

}  // namespace

cudaError_t launch_swa_prefill_tc(const void* q, const void* k, const void* v, void* y, void* k_cache,
                                  void* v_cache, int B, int H, int N, int w, float scale, unsigned* status,
                                  unsigned debug, cudaStream_t stream) {
    const uint64_t BH = (uint64_t)B * H;
    CUtensorMap mq, mk, mv;
    if (!make_tmap_bf16_3d(&mq, q, HD, N, BH, HD, QT) || !make_tmap_bf16_3d(&mk, k, HD, N, BH, HD, KW) ||
        !make_tmap_bf16_3d(&mv, v, HD, N, BH, HD, KW))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(swa_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const dim3 grid((N + QT - 1) / QT, (unsigned)BH);
    const float scale_log2 = scale * 1.4426950408889634f;     // exp(x) = exp2(x * log2(e))
    using bf = __nv_bfloat16;
    swa_prefill_tc_kernel<<<grid, kThreads, SMEM_BYTES, stream>>>(
        mq, mk, mv, static_cast<const bf*>(k), static_cast<const bf*>(v), static_cast<bf*>(y),
        static_cast<bf*>(k_cache), static_cast<bf*>(v_cache), N, w, scale_log2, status, debug);
    return cudaGetLastError();
}

}  // namespace based

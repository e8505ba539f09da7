// Tensor-core (tcgen05 / TMEM) sliding-window softmax attention prefill, bf16, head dim 64, w <= 64.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), §4 "Local Exact Attention": exact softmax over the w most
// recent keys (the query's own position included), O(Nw) work.
//
// A tile is 128 consecutive queries [i0, i0 + 128) of one head. Every key those
// queries can see lies in the 192-key span [i0 - 64, i0 + 128), so a tile needs
// exactly one score block and one value block -- no running softmax:
//   TMA    Q [128 x 64], K and V [192 x 64] (128-byte swizzle; rows before the
//          sequence start or past its end arrive as zeros)
//   MMA    S = Q K^T              M=128 N=192 K=64   -> TMEM (192 columns)
//   CUDA   row i keeps only its band i0+i-w < j <= i0+i; p = exp(scale*(s - max)),
//          written back as bf16 P over the first 96 columns of S (in place)
//   MMA    O = P V                M=128 N=64 K=192   -> TMEM (A operand P in TMEM)
//   CUDA   y = O / l, l = the sum of the rounded p -> swizzled tile -> TMA store
// A warp's 32 query rows touch only 96 of the 192 score columns; it reads just
// those and writes zeros for the rest of its P row.
//
// The kernel is persistent and pipelined: one CTA per SM walks its tiles
// (tile = CTA + k * grid) with
//   warp 0      lane 0 issues the TMA loads into a 3-stage ring of {Q, K, V};
//   warp 1      allocates TMEM; lane 0 issues S = Q K^T of each tile;
//   warp 10     lane 0 issues O = P V of each tile once its softmax is done
//               (two issuing warps, because one thread keeps only about one
//               MMA per ~100 cycles in flight);
//   warps 2-5   softmax + epilogue of even tiles (TMEM buffer 0),
//   warps 6-9   the same for odd tiles (TMEM buffer 1); the epilogue warps also
//               copy the tile's share of the last w tokens from the shared-
//               memory stage into the ring KV cache (slot t mod w) and, on a
//               head's first tile, zero the slots a prompt shorter than w
//               never fills.
// Every hand-off is an mbarrier; every wait is bounded.
#include <cuda.h>
#include <math.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma_host.h"

namespace based {
namespace {

using namespace tc;

constexpr int QT = 128;              // queries per tile
constexpr int KW = 192;              // keys per tile: [i0 - 64, i0 + 128)
constexpr int HD = 64;               // head dim
constexpr int kStages = 3;           // {Q, K, V} ring depth
constexpr int kThreads = 352;

// Shared memory (offsets from a 1024-aligned base).
constexpr uint32_t Q_BYTES = QT * HD * 2;          // 16 KB
constexpr uint32_t KV_BYTES = KW * HD * 2;         // 24 KB each
constexpr uint32_t STAGE_BYTES = Q_BYTES + 2 * KV_BYTES;
constexpr uint32_t OFF_STAGE = 0;                  // [kStages] {Q, K, V}
constexpr uint32_t OFF_YS = kStages * STAGE_BYTES; // [2] y tiles, 128-byte swizzled
constexpr uint32_t OFF_BAR = OFF_YS + 2 * Q_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256 + 1024;   // + alignment slack
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
constexpr uint32_t TX_BYTES = STAGE_BYTES;

// TMEM: two buffers of {S / P (192 columns), O (64 columns)}.
constexpr uint32_t COL_S = 0;
constexpr uint32_t COL_O = 192;
constexpr uint32_t BUF_COLS = 256;
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_S = idesc_bf16_f32(128, KW, false, false);
constexpr uint32_t ID_O = idesc_bf16_f32(128, HD, false, true);

enum {
    BAR_FULL0, BAR_FULL1, BAR_FULL2,          // TMA -> MMA: stage s landed
    BAR_EMPTY0, BAR_EMPTY1, BAR_EMPTY2,       // MMA commit: stage s read (S and O done)
    BAR_SF0, BAR_SF1,                         // MMA commit: S of buffer b ready
    BAR_PF0, BAR_PF1,                         // softmax warps -> MMA: P of buffer b written
    BAR_OF0, BAR_OF1,                         // MMA commit: O of buffer b ready
    BAR_TE0, BAR_TE1,                         // softmax warps -> MMA: TMEM buffer b read (free)
    BAR_YR0, BAR_YR1,                         // softmax warps -> store thread: y tile b written
    BAR_YE0, BAR_YE1,                         // store thread -> softmax warps: the TMA store has read y tile b
    NUM_BARS
};

struct Ctx {
    uint32_t sbase;
    uint64_t* bars;
    volatile int* abort_flag;
    unsigned* status;
    int N, w, nqb, ntiles;
};

// 2^x by the hardware approximation (relative error about 2^-22, far below the
// bf16 rounding P goes through); 2^-inf = +0.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ bool wait_bar(const Ctx& cx, int bar, uint32_t parity) {
    return mbar_wait(&cx.bars[bar], parity, cx.abort_flag, cx.status);
}

// ------------------------------------------------------------------ TMA producer (warp 0, lane 0)
__device__ __forceinline__ void producer(const Ctx& cx, const CUtensorMap* tq, const CUtensorMap* tk,
                                         const CUtensorMap* tv) {
    int n = 0;
    for (int tile = blockIdx.x; tile < cx.ntiles; tile += gridDim.x, ++n) {
        const int s = n % kStages;
        if (n >= kStages && !wait_bar(cx, BAR_EMPTY0 + s, ((n / kStages) - 1) & 1)) break;
        const int bh = tile / cx.nqb, i0 = (tile % cx.nqb) * QT;
        const uint32_t st = cx.sbase + OFF_STAGE + s * STAGE_BYTES;
        mbar_expect_tx(&cx.bars[BAR_FULL0 + s], TX_BYTES);
        tma_load_3d(st, tq, &cx.bars[BAR_FULL0 + s], 0, i0, bh);
        tma_load_3d(st + Q_BYTES, tk, &cx.bars[BAR_FULL0 + s], 0, i0 - 64, bh);
        tma_load_3d(st + Q_BYTES + KV_BYTES, tv, &cx.bars[BAR_FULL0 + s], 0, i0 - 64, bh);
    }
    // Loads still landing when the CTA ends would write freed shared memory:
    // wait (bounded) for the last ones.
    for (int m = max(0, n - kStages); m < n; ++m) {
        const uint64_t t0 = global_ns();
        while (!mbar_try_wait(&cx.bars[BAR_FULL0 + m % kStages], (m / kStages) & 1) && global_ns() - t0 < kWaitLimitNs) {}
    }
}

// ------------------------------------------------------------------ MMA issuers
// One thread keeps only about one tcgen05.mma per ~100 cycles in flight, so S
// and O come from two warps and overlap on the tensor core.

// Never free TMEM under an MMA still in flight: after an abort, wait (bounded)
// for the issuer's last commit.
__device__ __forceinline__ void drain(const Ctx& cx, uint64_t* last_bar, uint32_t last_parity) {
    if (!*cx.abort_flag || last_bar == nullptr) return;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(last_bar, last_parity) && global_ns() - t0 < kWaitLimitNs) {}
}

// S = Q K^T of every local tile n (warp 1, lane 0).
__device__ __forceinline__ void s_issuer(const Ctx& cx, uint32_t tmem) {
    uint64_t* last_bar = nullptr;
    uint32_t last_parity = 0;
    int n = 0;
    for (int tile = blockIdx.x; tile < cx.ntiles; tile += gridDim.x, ++n) {
        const int s = n % kStages, b = n & 1;
        if (!wait_bar(cx, BAR_FULL0 + s, (n / kStages) & 1)) break;
        if (n >= 2 && !wait_bar(cx, BAR_TE0 + b, ((n >> 1) - 1) & 1)) break;   // O of tile n-2 read out
        tc_fence_after();
        const uint32_t q = cx.sbase + OFF_STAGE + s * STAGE_BYTES;
        const uint32_t tb = tmem + b * BUF_COLS;
#pragma unroll
        for (int j = 0; j < HD / 16; ++j)
            mma_bf16(tb + COL_S, smem_desc_sw128(q + 32 * j, 16, 1024), smem_desc_sw128(q + Q_BYTES + 32 * j, 16, 1024),
                     ID_S, j > 0);
        mma_commit(&cx.bars[BAR_SF0 + b]);
        last_bar = &cx.bars[BAR_SF0 + b];
        last_parity = (n >> 1) & 1;
    }
    drain(cx, last_bar, last_parity);
}

// O = P V of every local tile n, once its softmax has written P (warp 10, lane 0).
__device__ __forceinline__ void o_issuer(const Ctx& cx, uint32_t tmem) {
    uint64_t* last_bar = nullptr;
    uint32_t last_parity = 0;
    int n = 0;
    for (int tile = blockIdx.x; tile < cx.ntiles; tile += gridDim.x, ++n) {
        const int s = n % kStages, b = n & 1;
        if (!wait_bar(cx, BAR_PF0 + b, (n >> 1) & 1)) break;
        tc_fence_after();
        const uint32_t v = cx.sbase + OFF_STAGE + s * STAGE_BYTES + Q_BYTES + KV_BYTES;
        const uint32_t tb = tmem + b * BUF_COLS;
#pragma unroll
        for (int j = 0; j < KW / 16; ++j)
            mma_bf16_ts(tb + COL_O, tb + COL_S + 8 * j, smem_desc_sw128(v + j * 2048, 16, 1024), ID_O, j > 0);
        mma_commit(&cx.bars[BAR_EMPTY0 + s]);     // S and O of tile n have read the stage
        mma_commit(&cx.bars[BAR_OF0 + b]);
        last_bar = &cx.bars[BAR_OF0 + b];
        last_parity = (n >> 1) & 1;
    }
    drain(cx, last_bar, last_parity);
}

// ------------------------------------------------------------------ softmax + epilogue (warps 2-9)
// Warpgroup g takes the tiles of TMEM buffer g; thread = query row i = TMEM lane
// (quadrant q = warp mod 4). The warp with quadrant 0 has the store thread.
__device__ __forceinline__ void softmax_wg(const Ctx& cx, uint32_t tmem, int g, int q, int lane,
                                           const CUtensorMap* ty, const __nv_bfloat16* __restrict__ k,
                                           const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ k_cache,
                                           __nv_bfloat16* __restrict__ v_cache, float scale_log2) {
    const int i = q * 32 + lane;
    const bool store_thread = q == 0 && lane == 0;
    const uint32_t lane_base = tmem + g * BUF_COLS + (static_cast<uint32_t>(q * 32) << 16);
    const uint32_t ys = cx.sbase + OFF_YS + g * Q_BYTES;
    const int N = cx.N, w = cx.w;
    int kk = 0;                                  // tiles of this warpgroup so far
    for (int tile = blockIdx.x + g * gridDim.x; tile < cx.ntiles; tile += 2 * gridDim.x, ++kk) {
        const int bh = tile / cx.nqb, i0 = (tile % cx.nqb) * QT, kb = i0 - 64, qi = i0 + i;
        if (!wait_bar(cx, BAR_SF0 + g, kk & 1)) return;
        tc_fence_after();
        // Columns [32q, 32q + 96) of S hold every key of this warp's rows.
        float sc[96];
#pragma unroll
        for (int m = 0; m < 6; ++m) tmem_ld16(lane_base + COL_S + 32 * q + 16 * m, sc + 16 * m);
        tmem_ld_wait();
        // This row's keys within the loaded window c = 0..95 (span column 32q + c)
        // form the contiguous range [lo, hi]: the band i - w < j <= i, cut at the
        // sequence start; a padding row (qi >= N) sees nothing.
        const int lo = max(lane + 65 - w, -kb - 32 * q);
        const int hi = qi < N ? lane + 64 : -1;
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 96; ++c) {
            sc[c] = (c >= lo && c <= hi) ? sc[c] : -INFINITY;
            mx = fmaxf(mx, sc[c]);
        }
        // p = exp(scale (s - max)) = 2^(s * scale_log2 - max * scale_log2); exp2 of
        // -inf is 0, so masked keys need no branch.
        const float off = mx == -INFINITY ? 0.f : -mx * scale_log2;
        // P row i in bf16 pairs over S: key pair (2m, 2m+1) of the span in column m.
        // Column groups q..q+2 (16 columns each) hold the band, the rest are zero.
        float l = 0.f;
        uint32_t pw[48];
#pragma unroll
        for (int m = 0; m < 48; ++m) {
            const uint32_t u = pack_bf16x2(ex2_approx(fmaf(sc[2 * m], scale_log2, off)),
                                           ex2_approx(fmaf(sc[2 * m + 1], scale_log2, off)));
            l += __uint_as_float(u << 16) + __uint_as_float(u & 0xFFFF0000u);   // the values the MMA will see
            pw[m] = u;
        }
        uint32_t zero[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) zero[e] = 0u;
#pragma unroll
        for (int gr = 0; gr < 6; ++gr) {
            const int rel = gr - q;              // warp-uniform
            if (rel == 0) tmem_st16(lane_base + COL_S + 16 * gr, pw);
            else if (rel == 1) tmem_st16(lane_base + COL_S + 16 * gr, pw + 16);
            else if (rel == 2) tmem_st16(lane_base + COL_S + 16 * gr, pw + 32);
            else tmem_st16(lane_base + COL_S + 16 * gr, zero);
        }
        tmem_st_wait();
        // Ring cache: token u in [max(0, N - w), N) goes to slot u mod w. Its K
        // and V rows are span rows i + 64 of this tile's stage, which stays
        // ours until O = P V (issued after PF) has completed; the stage data is
        // read here (its TMA has completed: FULL of this stage, this phase),
        // not from global memory, which cost the last tile of every head a
        // dependent round trip.
        if (k_cache != nullptr && i0 + QT > N - w) {
            const int n = 2 * kk + g, s = n % kStages;
            if (!wait_bar(cx, BAR_FULL0 + s, (n / kStages) & 1)) return;
            if (qi < N && qi >= N - w && in_bounds(((size_t)bh * w + qi % w) * HD + HD - 1,
                                                   (size_t)(cx.ntiles / cx.nqb) * w * HD, cx.status)) {
                const uint32_t kr = cx.sbase + OFF_STAGE + s * STAGE_BYTES + Q_BYTES + (i + 64) * 128;
                const uint32_t sw = (uint32_t)((i + 64) & 7);
                uint4* kd = reinterpret_cast<uint4*>(k_cache + ((size_t)bh * w + qi % w) * HD);
                uint4* vd = reinterpret_cast<uint4*>(v_cache + ((size_t)bh * w + qi % w) * HD);
#pragma unroll
                for (int p8 = 0; p8 < HD / 8; ++p8) {
                    kd[p8] = ld_shared_v4(kr + ((p8 ^ sw) << 4));
                    vd[p8] = ld_shared_v4(kr + KV_BYTES + ((p8 ^ sw) << 4));
                }
            }
        }
        tc_fence_before();
        mbar_arrive(&cx.bars[BAR_PF0 + g]);

        if (!wait_bar(cx, BAR_OF0 + g, kk & 1)) return;
        tc_fence_after();
        float o[HD];
#pragma unroll
        for (int m = 0; m < HD / 16; ++m) tmem_ld16(lane_base + COL_O + 16 * m, o + 16 * m);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&cx.bars[BAR_TE0 + g]);

        // y tile: free once the previous TMA store from it has read it.
        if (kk >= 1) {
            if (store_thread) {
                bulk_wait_read_all();
                mbar_arrive(&cx.bars[BAR_YE0 + g]);
            }
            if (!wait_bar(cx, BAR_YE0 + g, (kk - 1) & 1)) return;
        }
        const float inv = 1.0f / (l > 0.f ? l : 1.0f);
#pragma unroll
        for (int p8 = 0; p8 < HD / 8; ++p8) {
            float t[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) t[e] = o[8 * p8 + e] * inv;
            st_shared_v4(ys + i * 128 + ((p8 ^ (i & 7)) << 4), pack_bf16x8(t));
        }
        fence_proxy_async_smem();
        mbar_arrive(&cx.bars[BAR_YR0 + g]);
        if (store_thread) {
            if (!wait_bar(cx, BAR_YR0 + g, kk & 1)) return;
            tma_store_3d(ty, ys, 0, i0, bh);
            bulk_commit();
        }

        // Ring cache: a head's first tile zeroes the slots a prompt shorter than
        // w never fills (the filled slots were written before PF).
        if (k_cache != nullptr) {
            const size_t ring = (size_t)bh * w;
            if (i0 == 0 && N + i < w &&
                in_bounds((ring + N + i) * HD + HD - 1, (size_t)(cx.ntiles / cx.nqb) * w * HD, cx.status)) {
                uint4* kd = reinterpret_cast<uint4*>(k_cache + (ring + N + i) * HD);
                uint4* vd = reinterpret_cast<uint4*>(v_cache + (ring + N + i) * HD);
#pragma unroll
                for (int p8 = 0; p8 < HD / 8; ++p8) kd[p8] = vd[p8] = make_uint4(0, 0, 0, 0);
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
swa_prefill_tc_kernel(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                      const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap ty,
                      const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
                      __nv_bfloat16* __restrict__ k_cache, __nv_bfloat16* __restrict__ v_cache, int N, int w,
                      int nqb, int ntiles, float scale_log2, unsigned* status, unsigned debug) {
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw = smem_u32(smem_raw);
    const uint32_t sbase = (raw + 1023u) & ~1023u;
    unsigned char* smem = smem_raw + (sbase - raw);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_BAR + 8 * NUM_BARS + 4);
    const Ctx cx{sbase, bars, abort_flag, status, N, w, nqb, ntiles};

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    if (tid == 0) {
        for (int b = 0; b < NUM_BARS; ++b) {
            const bool group = (b >= BAR_PF0 && b <= BAR_PF1) || (b >= BAR_TE0 && b <= BAR_TE1) ||
                               (b >= BAR_YR0 && b <= BAR_YR1);
            mbar_init(&bars[b], group ? 128 : 1);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 1) tmem_alloc(tmem_slot, TMEM_COLS);
    const bool skip_mma = (debug & DEBUG_SKIP_MMA) != 0;     // testing: issue nothing, every waiter times out
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    grid_dependency_wait();                                  // inputs may come from the previous kernel

    if (warp == 0) {
        if (lane == 0) producer(cx, &tq, &tk, &tv);
    } else if (warp == 1) {
        if (lane == 0 && !skip_mma) s_issuer(cx, tmem);
    } else if (warp == 10) {
        if (lane == 0 && !skip_mma) o_issuer(cx, tmem);
    } else {
        const int g = (warp - 2) >> 2;
        softmax_wg(cx, tmem, g, warp & 3, lane, &ty, k, v, k_cache, v_cache, scale_log2);
        if ((warp & 3) == 0 && lane == 0) bulk_wait_all();   // the y stores have completed
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
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
    CUtensorMap mq, mk, mv, my;
    if (!make_tmap_bf16_3d(&mq, q, HD, N, BH, HD, QT) || !make_tmap_bf16_3d(&mk, k, HD, N, BH, HD, KW) ||
        !make_tmap_bf16_3d(&mv, v, HD, N, BH, HD, KW) || !make_tmap_bf16_3d(&my, y, HD, N, BH, HD, QT))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(swa_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 0;
    if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    const int nqb = (N + QT - 1) / QT;
    const long long ntiles = (long long)nqb * (long long)BH;
    if (ntiles > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
    const int grid = (int)std::min<long long>(ntiles, (long long)sms);
    const float scale_log2 = scale * 1.4426950408889634f;     // exp(x) = exp2(x * log2(e))
    using bf = __nv_bfloat16;
    return launch_pdl(swa_prefill_tc_kernel, dim3(grid), dim3(kThreads), SMEM_BYTES, stream, mq, mk, mv, my,
                      static_cast<const bf*>(k), static_cast<const bf*>(v), static_cast<bf*>(k_cache),
                      static_cast<bf*>(v_cache), N, w, nqb, (int)ntiles, scale_log2, status, debug);
}

}  // namespace based

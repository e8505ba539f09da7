// Tensor-core (tcgen05 / TMEM) chunked prefill of causal Taylor linear attention.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), App. B "Forward / Generation Prefill": the feature map and
// the causal dot product are computed together, tile by tile; a tile's output is
// a quadratic on-diagonal part under a local causal mask plus a linear
// off-diagonal part read from the cumulative state of earlier tiles. With the
// K-state normalisation (App. D.4), for a chunk c of C = 128 tokens:
//
//   s      = Q_c K_c^T                                MMA1  M=128 N=128 K=16
//   Y      = phi(Q_c) [S | z]_{c-1}                   MMA3  M=128 N=80 K=160 (A from TMEM)
//   [S|z] += phi(K_c)^T [V_c | 1]                     MMA4  two 128-row tiles, N=80, K=128,
//                                                           accumulated in TMEM across chunks (fp32)
//   A      = mask(1 + s + s^2/2)                      CUDA cores, from TMEM
//   Y     += A [V_c | 1]                              MMA2  M=128 N=80 K=128
//   y_c    = Y[:, :64] / Y[:, 64]                     epilogue
//
// The ones column appended to V makes every product carry its own
// denominator: A [V | 1] gives the row sums of A, phi(Q)[S | z] gives phi(q).z,
// and phi(K)^T [V | 1] gives the increment of z.
//
// phi never reaches HBM: each token's thread forms phi(q_t) and phi(k_t) in
// registers; phi(Q) goes straight into tensor memory (the A operand of MMA3),
// phi(K)^T into shared memory. The order-2 block is folded by symmetry,
// (q.k)^2/2 = sum_a (q_a^2/sqrt2)(k_a^2/sqrt2) + sum_{a<b} (q_a q_b)(k_a k_b),
// giving 1 + 16 + 136 = 153 features (padded to 160) instead of 273; the final
// state is expanded back to the 273-row layout on the way out.
//
// Segments ("recurrent across chunks", "Gated Slot Attention" App. A.1): when
// there are fewer (b, h) pairs than SMs, each sequence is cut into segments of
// whole chunks. A first launch (totals pass) runs only the state update over
// every segment but the last and stores each segment's [S | z] total in the
// caller's workspace; the main launch then starts segment s from the sum of
// the totals of segments 0..s-1, so all segments of a sequence run at once.
//
// One CTA per (b, h, segment) with four roles (416 threads), so that the
// tensor pipe, the CUDA cores and the memory system work on different chunks:
//   warps 0-3   producers: thread t loads token t of chunk c+1 (prefetched in
//               registers a chunk ahead) and writes Q, K, [V|1] and phi(K)^T
//               into the free half of the double-buffered shared-memory tiles,
//               then phi(Q) into tensor memory once MMA3 of the previous chunk
//               has consumed it.
//   warps 4-7   state: after each chunk, read the fp32 state rows 0..127 from
//               TMEM in one batch and publish them as the bf16 B operand of the
//               next MMA3 (double-buffered in shared memory); write the final
//               state (or the segment total).
//   warps 8-11  intra + epilogue: turn s into A and Y into y (TMEM lane = token);
//               warp 8, whose rows of A are the shortest, also publishes state
//               rows 128..159.
//   warp 12     allocates TMEM; lane 0 issues every MMA and commit in the order
//               MMA1, MMA3, MMA4, MMA2 so the CUDA-core stages (A, state
//               publication) overlap the long MMAs.
// Every hand-off is an mbarrier; every wait is bounded.
//
// Shared-memory operands use the canonical no-swizzle layouts (8-row x 16-byte
// core matrices, each a contiguous 128-byte block); each thread writes whole
// 16-byte rows of core matrices, so eight consecutive threads fill one block.
#include <algorithm>

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
constexpr int kThreads = 416;

// Shared memory map (bytes); [b] tiles are double-buffered by chunk parity.
// MMA4's second 128-row tile of phi(K)^T reads feature rows 128..255 of which
// only 128..159 exist; the rows beyond alias the next region (their products
// land in TMEM lanes that are never read).
constexpr uint32_t PK_BYTES = KF * C * 2;
constexpr uint32_t VA_BYTES = C * NV * 2;
constexpr uint32_t QK_BYTES = C * DF * 2;
constexpr uint32_t SB_BYTES = KF * NV * 2;
constexpr uint32_t OFF_PK = 0;                                  // [2] phi(K)^T: M=feature, K=token, MN-major
constexpr uint32_t OFF_VA = OFF_PK + 2 * PK_BYTES;              // [2] [V|1]: N=column, K=token, MN-major
constexpr uint32_t OFF_Q = OFF_VA + 2 * VA_BYTES;               // [2] Q: M=token, K=d', K-major
constexpr uint32_t OFF_K = OFF_Q + 2 * QK_BYTES;                // [2] K: N=token, K=d', K-major
constexpr uint32_t OFF_A = OFF_K + 2 * QK_BYTES;                // A: M=token i, K=token j, K-major
constexpr uint32_t OFF_SB = OFF_A + C * C * 2;                  // [2] [S|z] bf16: N=column, K=feature, MN-major
constexpr uint32_t OFF_BAR = OFF_SB + 2 * SB_BYTES;
constexpr uint32_t SMEM_BYTES = OFF_BAR + 256;
static_assert(OFF_PK + PK_BYTES + (2 * C / 8 - 1) * 128 + (C / 8 - 1) * (KF / 8) * 128 + 128 <= SMEM_BYTES,
              "second update tile must stay inside shared memory");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");

// Core-matrix strides (bytes) of each operand: {K direction, M/N direction}.
constexpr uint32_t PK_LBO = (KF / 8) * 128, PK_SBO = 128;
constexpr uint32_t A_LBO = 128, A_SBO = (C / 8) * 128;
constexpr uint32_t VA_LBO = (NV / 8) * 128, VA_SBO = 128;
constexpr uint32_t SB_LBO = (NV / 8) * 128, SB_SBO = 128;
constexpr uint32_t QK_LBO = 128, QK_SBO = (DF / 8) * 128;

// TMEM columns. Every region starts on a multiple of 32 columns (an accumulator
// at an unaligned column is a misaligned-address error).
constexpr uint32_t COL_S = 0;      // s = Q K^T, 128 fp32 columns
constexpr uint32_t COL_Y = 128;    // Y, 80 fp32 columns
constexpr uint32_t COL_PQ = 224;   // phi(Q), 160 bf16 = 80 columns
constexpr uint32_t COL_D0 = 320;   // [S|z] rows 0..127, 80 fp32 columns
constexpr uint32_t COL_D1 = 416;   // [S|z] rows 128..255, 80 fp32 columns
constexpr uint32_t TMEM_COLS = 512;

constexpr uint32_t ID_QK = idesc_bf16_f32(128, 128, false, false);
constexpr uint32_t ID_AV = idesc_bf16_f32(128, NV, false, true);
constexpr uint32_t ID_UPD = idesc_bf16_f32(128, NV, true, true);
constexpr uint32_t ID_INT = idesc_bf16_f32(128, NV, false, true);

// Floats of one segment total in the workspace: KF rows of [S | z] (NV columns).
constexpr size_t kTotalFloats = (size_t)KF * NV;

// Barriers: IN/FREE/SBF per buffer, the rest once per chunk (INIT and DONE once).
enum {
    BAR_IN0, BAR_IN1,        // producers -> MMA: Q, K, [V|1], phi(K)^T of a chunk are in buffer b
    BAR_FREE0, BAR_FREE1,    // MMA commit: every MMA reading buffer b has completed
    BAR_PQIN,                // producers -> MMA: phi(Q) is in TMEM
    BAR_PQF,                 // MMA commit: MMA3 done (phi(Q) free)
    BAR_SBF0, BAR_SBF1,      // MMA commit: MMA3 done reading [S|z] bf16 buffer b
    BAR_S,                   // MMA commit: s ready
    BAR_A,                   // epilogue warps -> MMA: A written
    BAR_DS,                  // MMA commit: MMA4 done, [S|z] in TMEM is the state after chunk c
    BAR_DSF,                 // state readers -> MMA: [S|z] read from TMEM
    BAR_SBR,                 // state readers -> MMA: [S|z] bf16 written
    BAR_Y,                   // MMA commit: Y complete
    BAR_YF,                  // epilogue warps -> MMA: Y read
    BAR_INIT,                // state readers -> MMA: start state of the segment is in TMEM and buffer 1
    BAR_DONE,                // MMA commit after the last MMA4 (totals pass)
    NUM_BARS
};

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

// Feature rows of the final state: folded row f maps to one or two rows of the
// 1 + d' + d'^2 layout (off-diagonal pairs are split evenly, each times 1/sqrt2).
__device__ __forceinline__ void write_state_row(float* S, float* z, size_t bh, int f, const float* Sr) {
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
            dst[j] = make_float4(Sr[4 * j] * coef, Sr[4 * j + 1] * coef, Sr[4 * j + 2] * coef, Sr[4 * j + 3] * coef);
        z[bh * feature_dim(DF) + rows[i]] = Sr[DV] * coef;
    }
}

// Everything a CTA needs to know about its share of the work.
struct Work {
    size_t bh;               // (b, h)
    int seg, nseg;           // segment index, segments per sequence
    int t_begin, t_end;      // tokens [t_begin, t_end) of the sequence
    int nchunks;
    bool totals;             // totals pass: state update only, result to the workspace
    bool has_init;           // main pass, segment > 0: starts from the workspace prefix sum
    bool final_state;        // main pass, last segment: writes S and z
    float* ws_out;           // totals pass: this segment's total
    const float* ws_in;      // main pass: totals of this sequence's segments 0..seg-1
};

// Bf16 row f of [S|z] buffer b (the B operand of MMA3).
__device__ __forceinline__ void store_sb_row(uint32_t sbase, int b, int f, const float* r) {
    const uint32_t row = sbase + OFF_SB + b * SB_BYTES + (f & 7) * 16 + (f >> 3) * SB_LBO;
    const bool real = f < DS;
#pragma unroll
    for (int j = 0; j < NV / 8; ++j) {
        float t8[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) t8[e] = real ? r[8 * j + e] : 0.f;
        st_shared_v4(row + j * SB_SBO, pack_bf16x8(t8));
    }
}

// Segment start state: row f = sum of the totals of segments 0..seg-1, placed in
// the TMEM accumulator (fp32) and in [S|z] buffer 1 (bf16) for MMA3 of chunk 0.
__device__ __forceinline__ void init_state(const Work& w, int f, uint32_t taddr, uint32_t sbase, uint64_t* bars) {
    float r[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) r[i] = 0.f;
    for (int s = 0; s < w.seg; ++s) {
        const float4* src = reinterpret_cast<const float4*>(w.ws_in + s * kTotalFloats + (size_t)f * NV);
#pragma unroll
        for (int j = 0; j < NV / 4; ++j) {
            const float4 t = __ldg(src + j);
            r[4 * j] += t.x; r[4 * j + 1] += t.y; r[4 * j + 2] += t.z; r[4 * j + 3] += t.w;
        }
    }
#pragma unroll
    for (int m = 0; m < NV / 16; ++m) {
        uint32_t u[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(r[16 * m + i]);
        tmem_st16(taddr + 16 * m, u);
    }
    tmem_st_wait();
    store_sb_row(sbase, 1, f, r);
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(&bars[BAR_INIT]);
}

// Main pass, after MMA4 of chunk c: read one 80-column state row (fp32, TMEM lane
// of the calling thread) in a single batch, release it to MMA4 of chunk c+1, then
// publish it as bf16 row f of [S|z] buffer c&1 for MMA3 of chunk c+1 -- or, after
// the last chunk of the last segment, write it out as the final state.
// Whole-warp call.
__device__ __forceinline__ bool publish_state(const Work& w, int c, int f, uint32_t taddr, uint64_t* bars,
                                              uint32_t sbase, volatile int* abort_flag, unsigned* status,
                                              float* S, float* z) {
    if (!mbar_wait(&bars[BAR_DS], c & 1, abort_flag, status)) return false;
    tc_fence_after();
    float r[NV];
#pragma unroll
    for (int m = 0; m < NV / 16; ++m) tmem_ld16(taddr + 16 * m, r + 16 * m);
    tmem_ld_wait();
    tc_fence_before();
    mbar_arrive(&bars[BAR_DSF]);
    if (c + 1 < w.nchunks) {
        const int b = c & 1;
        // Buffer b still holds the state read by MMA3 of chunk c-1 (or, for a
        // segment with a start state, by MMA3 of chunk 0 when c == 1).
        const bool wait = w.has_init ? c >= 1 : c >= 2;
        const uint32_t parity = (w.has_init && (c & 1)) ? ((c >> 1) & 1) : (((c >> 1) - 1) & 1);
        if (wait && !mbar_wait(&bars[BAR_SBF0 + b], parity, abort_flag, status)) return false;
        store_sb_row(sbase, b, f, r);
        fence_proxy_async_smem();
        mbar_arrive(&bars[BAR_SBR]);
    } else if (w.final_state && S != nullptr && !*abort_flag) {
        write_state_row(S, z, w.bh, f, r);
    }
    return true;
}

// Totals pass: once the last MMA4 has landed, copy row f of the accumulated
// [S|z] (fp32) to this segment's slot in the workspace. Whole-warp call.
__device__ __forceinline__ void store_total(const Work& w, int f, uint32_t taddr, uint64_t* bars,
                                            volatile int* abort_flag, unsigned* status) {
    if (!mbar_wait(&bars[BAR_DONE], 0, abort_flag, status)) return;
    tc_fence_after();
    float r[NV];
#pragma unroll
    for (int m = 0; m < NV / 16; ++m) tmem_ld16(taddr + 16 * m, r + 16 * m);
    tmem_ld_wait();
    float4* dst = reinterpret_cast<float4*>(w.ws_out + (size_t)f * NV);
#pragma unroll
    for (int j = 0; j < NV / 4; ++j) dst[j] = make_float4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
}

struct Raw {          // one token's inputs: q, k (2 x 16 B each), v (8 x 16 B)
    uint4 q[2], k[2], v[8];
};

__device__ __forceinline__ void load_token(Raw& r, const __nv_bfloat16* q, const __nv_bfloat16* k,
                                           const __nv_bfloat16* v, size_t row, bool valid) {
    if (valid) {
        const uint4* qp = reinterpret_cast<const uint4*>(q + row * DF);
        const uint4* kp = reinterpret_cast<const uint4*>(k + row * DF);
        const uint4* vp = reinterpret_cast<const uint4*>(v + row * DV);
        r.q[0] = __ldg(qp); r.q[1] = __ldg(qp + 1);
        r.k[0] = __ldg(kp); r.k[1] = __ldg(kp + 1);
#pragma unroll
        for (int i = 0; i < 8; ++i) r.v[i] = __ldg(vp + i);
    } else {
        r.q[0] = r.q[1] = r.k[0] = r.k[1] = make_uint4(0, 0, 0, 0);
#pragma unroll
        for (int i = 0; i < 8; ++i) r.v[i] = make_uint4(0, 0, 0, 0);
    }
}

// mode 0: main pass over every segment; mode 1: totals pass over segments 0..nseg-2.
__global__ void __launch_bounds__(kThreads, 1)
la_prefill_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                     const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ y,
                     float* __restrict__ S, float* __restrict__ z, int N, int nseg, int seg_chunks, int mode,
                     float* __restrict__ ws, unsigned* status, unsigned debug) {
    extern __shared__ __align__(1024) unsigned char smem[];
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + OFF_BAR + 8 * NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_BAR + 8 * NUM_BARS + 4);
    const uint32_t sbase = smem_u32(smem);

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    Work w;
    w.totals = mode == 1;
    const int per_head = w.totals ? nseg - 1 : nseg;
    w.bh = blockIdx.x / per_head;
    w.seg = blockIdx.x % per_head;
    w.nseg = nseg;
    w.t_begin = w.seg * seg_chunks * C;
    w.t_end = min(N, w.t_begin + seg_chunks * C);
    w.nchunks = (w.t_end - w.t_begin + C - 1) / C;
    w.has_init = !w.totals && w.seg > 0;
    w.final_state = !w.totals && w.seg == nseg - 1;
    w.ws_out = w.totals ? ws + (w.bh * (nseg - 1) + w.seg) * kTotalFloats : nullptr;
    w.ws_in = w.has_init ? ws + w.bh * (nseg - 1) * kTotalFloats : nullptr;
    const int nchunks = w.nchunks;

    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) {
            const bool per_warpgroup = i == BAR_IN0 || i == BAR_IN1 || i == BAR_PQIN || i == BAR_A || i == BAR_YF;
            const bool state = i == BAR_DSF || i == BAR_SBR || i == BAR_INIT;   // warps 4-7 plus warp 8
            mbar_init(&bars[i], per_warpgroup ? 128 : state ? 160 : 1);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 12) tmem_alloc(tmem_base_slot, TMEM_COLS);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;

    if (warp < 4) {
        // ------------------------------------------------------------ producers
        const int t = tid;                                   // token within chunk == TMEM lane
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const uint32_t cm = (t & 7) * 16;                    // row within a core matrix
        const size_t row0 = w.bh * (size_t)N;
        Raw nxt;
        load_token(nxt, q, k, v, row0 + w.t_begin + t, w.t_begin + t < w.t_end);
        for (int c = 0; c < nchunks; ++c) {
            const int b = c & 1;
            const int tok = w.t_begin + c * C + t;
            const bool valid = tok < w.t_end;
            const Raw cur = nxt;
            if (c + 1 < nchunks) load_token(nxt, q, k, v, row0 + tok + C, tok + C < w.t_end);
            if (c >= 2 && !mbar_wait(&bars[BAR_FREE0 + b], ((c >> 1) - 1) & 1, abort_flag, status)) break;
            // [V | 1] (MN-major: a 16-byte piece is 8 columns of token t)
            const uint32_t va = sbase + OFF_VA + b * VA_BYTES + cm + (t >> 3) * VA_LBO;
#pragma unroll
            for (int i = 0; i < 8; ++i) st_shared_v4(va + i * VA_SBO, cur.v[i]);
            st_shared_v4(va + 8 * VA_SBO, make_uint4(valid ? 0x3F80u : 0u, 0u, 0u, 0u));  // bf16 1.0, column 64
            st_shared_v4(va + 9 * VA_SBO, make_uint4(0, 0, 0, 0));
            // phi(K)^T (MN-major columns); padded tokens contribute nothing
            const uint32_t pk = sbase + OFF_PK + b * PK_BYTES + cm + (t >> 3) * PK_LBO;
            if (valid) {
                float xk[DF];
                unpack_bf16x8(cur.k[0], xk);
                unpack_bf16x8(cur.k[1], xk + 8);
                emit_phi(xk, [&](int j, uint4 u) { st_shared_v4(pk + j * PK_SBO, u); });
            } else {
#pragma unroll
                for (int j = 0; j < KF / 8; ++j) st_shared_v4(pk + j * PK_SBO, make_uint4(0, 0, 0, 0));
            }
            if (!w.totals) {
                // Q, K (K-major, 2 core matrices along d')
                const uint32_t qk = cm + (t >> 3) * QK_SBO + b * QK_BYTES;
                st_shared_v4(sbase + OFF_Q + qk, cur.q[0]);
                st_shared_v4(sbase + OFF_Q + qk + QK_LBO, cur.q[1]);
                st_shared_v4(sbase + OFF_K + qk, cur.k[0]);
                st_shared_v4(sbase + OFF_K + qk + QK_LBO, cur.k[1]);
            }
            fence_proxy_async_smem();
            mbar_arrive(&bars[BAR_IN0 + b]);
            if (w.totals) continue;

            // phi(Q) -> TMEM lane t, once MMA3 of the previous chunk has read it
            float xq[DF];
            unpack_bf16x8(cur.q[0], xq);
            unpack_bf16x8(cur.q[1], xq + 8);
            if (c >= 1 && !mbar_wait(&bars[BAR_PQF], (c - 1) & 1, abort_flag, status)) break;
            tc_fence_after();
            uint32_t pkt[16];
            emit_phi(xq, [&](int j, uint4 u) {
                pkt[(j & 3) * 4 + 0] = u.x;
                pkt[(j & 3) * 4 + 1] = u.y;
                pkt[(j & 3) * 4 + 2] = u.z;
                pkt[(j & 3) * 4 + 3] = u.w;
                if ((j & 3) == 3) tmem_st16(lane_base + COL_PQ + (j >> 2) * 16, pkt);
            });
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&bars[BAR_PQIN]);
        }
    } else if (warp < 8) {
        // ------------------------------------------------------------ state rows 0..127
        const int f = (warp - 4) * 32 + lane;                // folded feature row == TMEM lane
        const uint32_t taddr = tmem + (static_cast<uint32_t>((warp - 4) * 32) << 16) + COL_D0;
        if (w.totals) {
            store_total(w, f, taddr, bars, abort_flag, status);
        } else {
            if (w.has_init) init_state(w, f, taddr, sbase, bars);
            for (int c = 0; c < nchunks; ++c)
                if (!publish_state(w, c, f, taddr, bars, sbase, abort_flag, status, S, z)) break;
        }
    } else if (warp < 12) {
        // ------------------------------------------------------------ intra + epilogue
        const int wq = warp - 8;
        const int t = wq * 32 + lane;                        // token within chunk == TMEM lane
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
        const uint32_t a_off = OFF_A + (t & 7) * 16 + (t >> 3) * A_SBO;
        if (w.totals) {
            if (wq == 0) store_total(w, 128 + lane, lane_base + COL_D1, bars, abort_flag, status);
        } else {
            if (wq == 0 && w.has_init) init_state(w, 128 + lane, lane_base + COL_D1, sbase, bars);
            for (int c = 0; c < nchunks; ++c) {
                if (!mbar_wait(&bars[BAR_S], c & 1, abort_flag, status)) break;
                tc_fence_after();
                // Row t of A: columns above the warp's diagonal block are zero; the
                // rest come from TMEM in at most two batches of 64 columns.
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    if (2 * half > wq) {
#pragma unroll
                        for (int j = 0; j < 8; ++j)
                            st_shared_v4(sbase + a_off + (8 * half + j) * A_LBO, make_uint4(0, 0, 0, 0));
                        continue;
                    }
                    const bool two = 2 * half + 1 <= wq;     // second 32-column block also needed
                    float s[64];
#pragma unroll
                    for (int m = 0; m < 2; ++m) tmem_ld16(lane_base + COL_S + 64 * half + 16 * m, s + 16 * m);
                    if (two) {
#pragma unroll
                        for (int m = 2; m < 4; ++m) tmem_ld16(lane_base + COL_S + 64 * half + 16 * m, s + 16 * m);
                    }
                    tmem_ld_wait();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        if (j >= 4 && !two) {
                            st_shared_v4(sbase + a_off + (8 * half + j) * A_LBO, make_uint4(0, 0, 0, 0));
                            continue;
                        }
                        float a8[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int col = 64 * half + 8 * j + e;
                            const float sv = s[8 * j + e];
                            a8[e] = col <= t ? fmaf(sv, fmaf(0.5f, sv, 1.0f), 1.0f) : 0.0f;
                        }
                        st_shared_v4(sbase + a_off + (8 * half + j) * A_LBO, pack_bf16x8(a8));
                    }
                }
                fence_proxy_async_smem();
                tc_fence_before();
                mbar_arrive(&bars[BAR_A]);

                // state rows 128..159 (TMEM lanes 0..31 of the second tile): warp 8
                if (wq == 0 && !publish_state(w, c, 128 + lane, lane_base + COL_D1, bars, sbase, abort_flag,
                                              status, S, z))
                    break;

                if (!mbar_wait(&bars[BAR_Y], c & 1, abort_flag, status)) break;
                tc_fence_after();
                float yv[NV];
#pragma unroll
                for (int m = 0; m < NV / 16; ++m) tmem_ld16(lane_base + COL_Y + 16 * m, yv + 16 * m);
                tmem_ld_wait();
                tc_fence_before();
                mbar_arrive(&bars[BAR_YF]);
                const int tok = w.t_begin + c * C + t;
                if (tok < w.t_end) {
                    const float inv = 1.0f / yv[DV];
                    uint4* yp = reinterpret_cast<uint4*>(y + (w.bh * (size_t)N + tok) * DV);
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        float o[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) o[e] = yv[8 * i + e] * inv;
                        yp[i] = pack_bf16x8(o);
                    }
                }
            }
        }
    } else if (lane == 0) {
        // ------------------------------------------------------------ MMA issuer
        // Descriptors of buffer 0; buffer 1 and the K steps are byte offsets added
        // to the start-address field (addresses stay below 256 KB, so no carry).
        const uint64_t dq0 = smem_desc(sbase + OFF_Q, QK_LBO, QK_SBO);
        const uint64_t dk0 = smem_desc(sbase + OFF_K, QK_LBO, QK_SBO);
        const uint64_t dpk0 = smem_desc(sbase + OFF_PK, PK_LBO, PK_SBO);
        const uint64_t dva0 = smem_desc(sbase + OFF_VA, VA_LBO, VA_SBO);
        const uint64_t dsb0 = smem_desc(sbase + OFF_SB, SB_LBO, SB_SBO);
        const uint64_t da0 = smem_desc(sbase + OFF_A, A_LBO, A_SBO);
        uint64_t* last_bar = nullptr;
        uint32_t last_parity = 0;
        bool ok = !(debug & DEBUG_SKIP_MMA);                // testing: issue nothing, every waiter times out
        if (ok && w.has_init) ok = mbar_wait(&bars[BAR_INIT], 0, abort_flag, status);
        for (int c = 0; ok && c < nchunks; ++c) {
            const int b = c & 1;
            if (!mbar_wait(&bars[BAR_IN0 + b], (c >> 1) & 1, abort_flag, status)) break;
            tc_fence_after();
            const uint64_t dva = dva0 + ((b * VA_BYTES) >> 4);
            bool did_mma3 = false;
            if (!w.totals) {
                // MMA1: s = Q K^T
                mma_bf16(tmem + COL_S, dq0 + ((b * QK_BYTES) >> 4), dk0 + ((b * QK_BYTES) >> 4), ID_QK, 0);
                mma_commit(&bars[BAR_S]);
                // MMA3: Y = phi(Q) [S|z]_{c-1}
                if (!mbar_wait(&bars[BAR_PQIN], c & 1, abort_flag, status)) break;
                if (c > 0 || w.has_init) {
                    if (c > 0) {
                        if (!mbar_wait(&bars[BAR_YF], (c - 1) & 1, abort_flag, status)) break;
                        if (!mbar_wait(&bars[BAR_SBR], (c - 1) & 1, abort_flag, status)) break;
                    }
                    tc_fence_after();
                    const uint64_t dsb = dsb0 + ((((c - 1) & 1) * SB_BYTES) >> 4);
#pragma unroll
                    for (int j = 0; j < KF / 16; ++j)
                        mma_bf16_ts(tmem + COL_Y, tmem + COL_PQ + 8 * j, dsb + ((j * 2 * SB_LBO) >> 4), ID_INT, j > 0);
                    did_mma3 = true;
                }
                mma_commit(&bars[BAR_PQF]);
                if (did_mma3) mma_commit(&bars[BAR_SBF0 + ((c - 1) & 1)]);
                // MMA4 waits until the state readers are done with the previous state
                if (c > 0 && !mbar_wait(&bars[BAR_DSF], (c - 1) & 1, abort_flag, status)) break;
                tc_fence_after();
            }
            // MMA4: [S|z] += phi(K)^T [V|1]
            const uint64_t dpk = dpk0 + ((b * PK_BYTES) >> 4);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
#pragma unroll
                for (int j = 0; j < C / 16; ++j)
                    mma_bf16(tmem + (r == 0 ? COL_D0 : COL_D1), dpk + ((r * 16 * PK_SBO + j * 2 * PK_LBO) >> 4),
                             dva + ((j * 2 * VA_LBO) >> 4), ID_UPD, (c > 0 || j > 0 || w.has_init) ? 1u : 0u);
            }
            if (!w.totals) {
                mma_commit(&bars[BAR_DS]);
                // MMA2: Y += A [V|1]
                if (!mbar_wait(&bars[BAR_A], c & 1, abort_flag, status)) break;
                tc_fence_after();
#pragma unroll
                for (int j = 0; j < C / 16; ++j)
                    mma_bf16(tmem + COL_Y, da0 + ((j * 2 * A_LBO) >> 4), dva + ((j * 2 * VA_LBO) >> 4), ID_AV,
                             (did_mma3 || j > 0) ? 1u : 0u);
                mma_commit(&bars[BAR_Y]);
                last_bar = &bars[BAR_Y];
                last_parity = c & 1;
            }
            mma_commit(&bars[BAR_FREE0 + b]);
            if (w.totals) {
                last_bar = &bars[BAR_FREE0 + b];
                last_parity = (c >> 1) & 1;
            }
        }
        if (w.totals && !*abort_flag && last_bar != nullptr) mma_commit(&bars[BAR_DONE]);
        // Never free TMEM under an MMA still in flight: on abort, wait (bounded) for the last commit.
        if (*abort_flag && last_bar != nullptr) {
            const uint64_t t0 = global_ns();
            while (!mbar_try_wait(last_bar, last_parity) && global_ns() - t0 < kWaitLimitNs) {}
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 12) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Segments per sequence: enough CTAs to cover the SMs once, whole chunks each.
void plan_segments(int BH, int N, int num_sms, int* nseg, int* seg_chunks) {
    const int nchunks = (N + C - 1) / C;
    int n = 1;
    if (BH < num_sms) n = std::min(nchunks, std::max(1, num_sms / BH));
    const int per = (nchunks + n - 1) / n;
    *seg_chunks = per;
    *nseg = (nchunks + per - 1) / per;
}

}  // namespace

bool la_prefill_tc_supported(int d_feat, int d_v, int chunk) {
    return d_feat == DF && d_v == DV && chunk == C;
}

size_t la_prefill_tc_workspace(int B, int H, int N, int d_feat, int d_v, int chunk, int num_sms) {
    if (!la_prefill_tc_supported(d_feat, d_v, chunk)) return 0;
    int nseg, seg_chunks;
    plan_segments(B * H, N, num_sms, &nseg, &seg_chunks);
    return (size_t)B * H * (nseg - 1) * kTotalFloats * sizeof(float);
}

cudaError_t launch_la_prefill_tc(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    if (!la_prefill_tc_supported(a.d_feat, a.d_v, a.chunk) || !a.bf16) return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(la_prefill_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)SMEM_BYTES);
    if (e != cudaSuccess) return e;
    const int BH = a.B * a.H;
    int nseg, seg_chunks;
    plan_segments(BH, a.N, num_sms, &nseg, &seg_chunks);
    using bf = __nv_bfloat16;
    auto q = static_cast<const bf*>(a.q);
    auto k = static_cast<const bf*>(a.k);
    auto v = static_cast<const bf*>(a.v);
    auto y = static_cast<bf*>(a.y);
    float* ws = static_cast<float*>(a.workspace);
    if (nseg > 1) {
        la_prefill_tc_kernel<<<BH * (nseg - 1), kThreads, SMEM_BYTES, stream>>>(
            q, k, v, y, a.S, a.z, a.N, nseg, seg_chunks, 1, ws, a.status, a.debug);
        e = cudaGetLastError();
        if (e != cudaSuccess) return e;
    }
    la_prefill_tc_kernel<<<BH * nseg, kThreads, SMEM_BYTES, stream>>>(q, k, v, y, a.S, a.z, a.N, nseg, seg_chunks, 0,
                                                                    ws, a.status, a.debug);
    return cudaGetLastError();
}

}  // namespace based

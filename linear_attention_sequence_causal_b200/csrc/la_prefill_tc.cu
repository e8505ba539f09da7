// Tensor-core (tcgen05 / TMEM) chunked prefill of causal Taylor linear attention.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), App. B "Forward / Generation Prefill": the feature map and
// the causal dot product are computed together, tile by tile; a tile's output is
// a quadratic on-diagonal part under a local causal mask plus a linear
// off-diagonal part read from the cumulative state of earlier chunks. With the
// K-state normalisation (App. D.4), for a tile t of 128 tokens (the M of every
// MMA below) inside a chunk of CL tokens:
//
//   s         = Q_t K_j^T                          MMA1  M=128 N=128 K=16
//   A         = mask(1 + s + s^2/2)                CUDA cores, TMEM -> TMEM (bf16, spare columns)
//   Y         = phi(Q_t) [S | z]_{chunk start}     MMA3  M=128 N=80  K=160 (A operand in TMEM)
//   Y        += A [V_j | 1]                        MMA2  M=128 N=80  K=128 (A operand in TMEM)
//   [S|z]^T  += [V_t | 1]^T phi(K_t)               MMA4  M=128 N=160 K=128, fp32 in TMEM
//   y_t       = Y[:, :64] / Y[:, 64]               epilogue
//
// The chunk length CL decides which pairs (query, key) go through the
// quadratic form (same chunk) and which through the state (earlier chunks):
//   CL = 128  one chunk per tile: j = t, causal mask; the state after each tile
//             is read out and published for the next tile's MMA3.
//   CL = 256  two tiles per chunk: an odd tile adds the full (unmasked) block
//             j = t-1 of its chunk, and its MMA3 reads the same state as the
//             even tile before it; the state is read out after odd tiles only.
//   CL = 64   two chunks per tile: the mask keeps each query's own chunk only
//             (block diagonal); MMA3 runs twice, for rows 0-63 with the state
//             before the tile and for rows 64-127 with the state after its
//             first 64 tokens (phi(Q) has the other half's rows zeroed for each
//             pass), and MMA4 is split at token 64 so that state is read out
//             in between.
// All three give the same sum up to rounding.
//
// The ones column appended to V makes every product carry its own
// denominator: A [V | 1] gives the row sums of A, phi(Q)[S | z] gives phi(q).z,
// and [V | 1]^T phi(K) gives the increment of z in its last row.
//
// phi never reaches HBM: each token's thread forms phi(q_t) and phi(k_t) in
// registers; phi(Q) goes straight into tensor memory, phi(K) into shared
// memory. The order-2 block is folded by symmetry,
// (q.k)^2/2 = sum_a (q_a^2/sqrt2)(k_a^2/sqrt2) + sum_{a<b} (q_a q_b)(k_a k_b),
// giving 1 + 16 + 136 = 153 features (padded to 160) instead of 273, in an
// order that suits packed bf16x2 multiplies (see emit_phi2); the final state is
// expanded back to the 273-row layout on the way out.
//
// Issue structure. One thread can keep only about one tcgen05.mma per ~117
// cycles in flight (measured on B200 for any N <= 144), while MMAs from two
// issuing warps into separate accumulators overlap. So two warps issue:
//   warp 13  the Y chain: MMA3, MMA2 of every block of the tile, MMA1 of the
//            next block;
//   warp 12  the state chain: MMA4 (8 instructions of N = 160 per tile; the
//            state is kept transposed -- TMEM lane = value column, column =
//            feature -- which halves the instruction count of the natural layout).
// A has its own tensor-memory columns, so MMA1 of the next block can overwrite
// s as soon as A has been formed, and the next A is computed while MMA2 still
// reads the previous one (only its stores wait for MMA2). Keeping A (and
// phi(Q)) in tensor memory matters: an MMA of N = 80 with both operands in
// shared memory is bound by shared-memory bandwidth (6.5 KB per 40 tensor cycles).
//
// Other roles (480 threads, one CTA per (b, h, segment)); a warp reaches the
// TMEM lanes of quadrant (warp mod 4):
//   warp 14     input loader: TMA loads of the Q, K and V tiles into a ring of
//               stages, in the layouts the MMAs read (Q, K rows of 32 bytes
//               under the 32-byte swizzle; V rows of 128 bytes under the
//               128-byte swizzle, with a constant ones block as the second
//               atom that makes it [V | 1]), a stage at a time as the MMAs
//               reading it complete.
//   warps 0-3   producers: thread t reads q_t and k_t from the landed stage
//               and writes phi(K) into the free one of two shared-memory
//               tiles, and phi(Q) into TMEM once MMA3 has consumed the
//               previous one.
//   warps 4-7   intra + state: turn s into A (TMEM lane = token); warps 4-6
//               also read the fp32 state after MMA4 (lane = value column,
//               0..79) and publish it as the bf16 B operand of the next MMA3,
//               and stage the final state or write a segment total.
//   warps 8-11  epilogue: turn Y into y (TMEM lane = token) in a 128-byte
//               swizzled shared-memory tile that one thread stores with TMA.
// Every hand-off is an mbarrier; every wait is bounded.
//
// Segments ("recurrent across chunks", "Gated Slot Attention" App. A.1): when
// there are fewer (b, h) pairs than SMs, each sequence is cut into segments of
// whole chunks. A first launch (totals pass) runs only the state chain over
// every segment but the last and stores each segment's [S | z] total in the
// workspace; a small launch turns them into running sums (the state entering
// each segment) and the main launch then starts segment s from that state, so
// all segments of a sequence run at once.
//
// phi(K) and the bf16 state use the canonical no-swizzle layouts (8-row x
// 16-byte core matrices, each a contiguous 128-byte block); each thread writes
// whole 16-byte rows of core matrices, so eight consecutive threads fill one block.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"
#include "tma_host.h"

namespace based {
namespace {

using namespace tc;

constexpr int DF = 16;           // feature dim d'
constexpr int DV = 64;           // value dim
constexpr int C = 128;           // tokens per tile (the M of every MMA)
constexpr int DS = 153;          // distinct (symmetric) features
constexpr int KF = 160;          // DS padded to the MMA K step
constexpr int NV = 80;           // [V | 1] padded to the MMA N step
constexpr int kThreads = 480;
constexpr int kStateLanes = 96;  // warps 4-6 read state lanes 0..95 (0..79 hold data)

// ------------------------------------------------------------------ shared memory
// phi(K) tiles are double-buffered by tile parity; the inputs Q, K, V arrive by
// TMA in a ring of stages(CL) stages, in the layouts the MMAs read directly.
__host__ __device__ constexpr int stages(int cl) { return cl == 64 ? 2 : 3; }
constexpr uint32_t PK_BYTES = C * KF * 2;       // phi(K): K = token, N = feature, MN-major (no swizzle)
constexpr uint32_t V_BYTES = C * DV * 2;        // V: rows = tokens of 64 values (128 B), 128-byte swizzle
constexpr uint32_t QK_BYTES = C * DF * 2;       // Q, K: rows = tokens of d' values (32 B), 32-byte swizzle
constexpr uint32_t SB_BYTES = KF * NV * 2;      // [S|z] bf16: N = column, K = feature, K-major (no swizzle)
constexpr uint32_t YS_BYTES = C * DV * 2;       // y tile, 128-byte swizzled rows (TMA store source)
constexpr uint32_t QK_SBO = 8 * DF * 2;         // 8-row atoms of the 32-byte swizzle
constexpr uint32_t OFF_PK = 0;                                  // [2]
constexpr uint32_t OFF_SB = OFF_PK + 2 * PK_BYTES;              // [S|z] of the state before the tile
constexpr uint32_t OFF_SB1 = OFF_SB + SB_BYTES;                 // CL = 64: the state after its first chunk
// The rest depends on the chunk length (a second [S|z] buffer and two input
// stages at CL = 64, three stages otherwise). The 128-byte swizzled tiles start
// on 1024-byte boundaries, the 32-byte swizzled ones on 256-byte boundaries.
__host__ __device__ constexpr uint32_t off_v(int cl) { return OFF_SB + (cl == 64 ? 2 : 1) * SB_BYTES; }
// The ones block: V's second 64-column atom (column 64 = 1, the rest 0, for
// every token), shared by all stages. With it, a V stage read as an operand of
// N (or M) > 64 is [V | 1 | 0...]: the descriptor's atom stride points here.
__host__ __device__ constexpr uint32_t off_ones(int cl) { return off_v(cl) + stages(cl) * V_BYTES; }
__host__ __device__ constexpr uint32_t off_q(int cl) { return off_ones(cl) + V_BYTES; }
__host__ __device__ constexpr uint32_t off_k(int cl) { return off_q(cl) + stages(cl) * QK_BYTES; }
__host__ __device__ constexpr uint32_t off_ys(int cl) {        // [2], 1024-aligned for the swizzle
    return (off_k(cl) + stages(cl) * QK_BYTES + 1023) & ~1023u;
}
__host__ __device__ constexpr uint32_t off_bar(int cl) { return off_ys(cl) + 2 * YS_BYTES; }
__host__ __device__ constexpr uint32_t smem_bytes(int cl) { return off_bar(cl) + 256; }
static_assert(smem_bytes(64) <= 227 * 1024 && smem_bytes(128) <= 227 * 1024, "shared memory");
// The totals pass reads neither Q nor an [S|z] operand, and its ring is the
// chain's latency: a tile's stage comes free only once its MMA4 has completed,
// and the next load into it then takes about a microsecond to land. So it runs
// kTotalsStages stages, the extra ones (K and V) in the idle [S|z] region.
constexpr int kTotalsStages = 4;
__host__ __device__ constexpr int ring(int cl, bool totals) { return totals ? kTotalsStages : stages(cl); }
__host__ __device__ constexpr int extra_stages(int cl) { return kTotalsStages - stages(cl); }
__device__ __forceinline__ uint32_t stage_v(int cl, bool totals, int s) {
    return !totals || s < stages(cl) ? off_v(cl) + s * V_BYTES : OFF_SB + (s - stages(cl)) * V_BYTES;
}
__device__ __forceinline__ uint32_t stage_k(int cl, bool totals, int s) {
    return !totals || s < stages(cl) ? off_k(cl) + s * QK_BYTES
                                     : OFF_SB + extra_stages(cl) * V_BYTES + (s - stages(cl)) * QK_BYTES;
}
static_assert(extra_stages(64) * (V_BYTES + QK_BYTES) <= 2 * SB_BYTES &&
                  extra_stages(128) * (V_BYTES + QK_BYTES) <= SB_BYTES && OFF_SB % 1024 == 0 &&
                  (OFF_SB + extra_stages(64) * V_BYTES) % 256 == 0 && (OFF_SB + extra_stages(128) * V_BYTES) % 256 == 0,
              "the totals pass's extra stages fit the [S|z] region (below the ones block), aligned");
static_assert(off_v(64) % 1024 == 0 && off_v(128) % 1024 == 0 && off_q(64) % 256 == 0 && off_q(128) % 256 == 0,
              "swizzled tiles aligned");

// Core-matrix strides (bytes) of the no-swizzle operands: LBO along K, SBO along M/N.
constexpr uint32_t PK_LBO = (KF / 8) * 128, PK_SBO = 128;
constexpr uint32_t SB_LBO = 128, SB_SBO = (KF / 8) * 128;

// ------------------------------------------------------------------ tensor memory
// Every region starts on a multiple of 32 columns (an accumulator at an
// unaligned column is a misaligned-address error).
constexpr uint32_t COL_S = 0;      // s = Q K^T, 128 fp32 columns
constexpr uint32_t COL_Y = 128;    // Y, 80 fp32 columns
constexpr uint32_t COL_PQ = 224;   // phi(Q), 160 bf16 = 80 columns
constexpr uint32_t COL_ST = 320;   // [S|z]^T: lane = value column, 160 fp32 columns = features
constexpr uint32_t TMEM_COLS = 512;
static_assert(COL_ST + KF <= TMEM_COLS, "tensor memory");
// A (bf16, two keys per column) in the columns the regions above leave free:
// key block kb (32 keys, 16 columns) at col_a(kb).
__host__ __device__ constexpr uint32_t col_a(int kb) {
    return kb == 0 ? 480u : kb == 1 ? 496u : kb == 2 ? COL_Y + NV : COL_PQ + KF / 2;
}
static_assert(COL_Y + NV + 16 <= COL_PQ && COL_PQ + KF / 2 + 16 <= COL_ST && COL_ST + KF + 32 <= TMEM_COLS,
              "A columns");

constexpr uint32_t ID_QK = idesc_bf16_f32(128, C, false, false);
constexpr uint32_t ID_AV = idesc_bf16_f32(128, NV, false, true);   // A in TMEM, [V|1] MN-major (V stage + ones)
constexpr uint32_t ID_INT = idesc_bf16_f32(128, NV, false, false);
constexpr uint32_t ID_UPD = idesc_bf16_f32(128, KF, true, true);

// Floats of one segment total in the workspace: NV value-column rows of KF features.
constexpr size_t kTotalFloats = (size_t)KF * NV;

enum {
    BAR_RF0, BAR_RF1, BAR_RF2, BAR_RF3,   // TMA: Q, K, V of a tile landed in input stage s
    BAR_RE0, BAR_RE1, BAR_RE2, BAR_RE3,   // both issuers' commits: every MMA reading input stage s has completed
    BAR_PKF0, BAR_PKF1,          // state-issuer commit: MMA4 has read phi(K) buffer b
    BAR_IN0, BAR_IN1,            // producers -> state issuer: phi(K) of a tile is in buffer b
    BAR_PQIN,                // producers -> Y issuer: phi(Q) (one MMA3 pass's rows) is in TMEM
    BAR_PQF,                 // Y-issuer commit: MMA3 (CL = 64: of rows 0-63) done; phi(Q) and the [S|z] buffer it read are free
    BAR_PQF_HI,              // CL = 64: the same for the MMA3 of rows 64-127
    BAR_S,                   // Y-issuer commit: s of a block ready
    BAR_A,                   // intra warps -> Y issuer: A of a block written (s has been read)
    BAR_AF,                  // Y-issuer commit: MMA2 of a block done (the A columns are free)
    BAR_Y,                   // Y-issuer commit: Y of a tile complete
    BAR_YF,                  // epilogue warps -> Y issuer: Y read
    BAR_DS,                  // state-issuer commit: MMA4 done, the TMEM state is the state to read out
    BAR_DSF,                 // state warps -> state issuer: fp32 state read
    BAR_SBR,                 // state warps -> Y issuer: [S|z] bf16 written (buffer OFF_SB)
    BAR_SBR1,                // CL = 64: the same for buffer OFF_SB1
    BAR_INIT,                // state warps -> issuers: start state of the segment is in TMEM and the [S|z] buffer
    BAR_INITLD,              // copy of the segment's start state (main pass, segment > 0) landed
    BAR_YSR0, BAR_YSR1,      // epilogue warps -> store thread: y tile b written
    BAR_YSF0, BAR_YSF1,      // store thread -> epilogue warps: the TMA store has read y tile b
    NUM_BARS
};
static_assert(8 * NUM_BARS + 8 <= 256, "barrier area");

// ------------------------------------------------------------------ chunk plan
// Tiles per chunk (CL >= 128) and chunks per tile (CL < 128); the MMA tile is
// always 128 tokens. A tile's position in its chunk, its intra blocks and its
// state read-outs follow from CL and the tile's index c in the segment
// (segments start on chunk boundaries).
template <int CL>
struct Plan {
    static_assert(CL == 64 || CL == 128 || CL == 256, "chunk length");
    static constexpr int kSteps = CL < C ? 2 : 1;       // MMA4 steps (and read-outs) per tile
    // Intra blocks of tile c: key tiles c - blocks(c) + 1 .. c.
    __device__ static int blocks(int c) { return CL == 256 ? 1 + (c & 1) : 1; }
    // Blocks of tiles 0..c-1.
    __device__ static int blocks_before(int c) { return CL == 256 ? c + (c >> 1) : c; }
    // Whether the state is read out after tile c (of ntiles): after every tile
    // but the first of a pair at CL = 256, and always after the last.
    __device__ static bool reads_after(int c, int ntiles) {
        return CL != 256 || (c & 1) || c + 1 == ntiles;
    }
    // Read-outs before tile c's.
    __device__ static int readouts_before(int c) { return CL == 256 ? (c >> 1) : kSteps * c; }
};

// ------------------------------------------------------------------ feature map
// Kernel-internal order of the 153 distinct features (padded to 160), chosen so
// that the order-2 products come out of packed bf16x2 multiplies of the bf16
// inputs (a product of two bf16 values is exact in fp32, so one bf16x2 multiply
// rounds exactly like an fp32 multiply followed by a bf16 conversion):
//   0..15    x_a                                   (the input words themselves)
//   16..31   x_a^2 / sqrt2                         (fp32, then bf16)
//   32..143  x_a x_b for b = 2..15, a < 2 floor(b/2), by column b, pairs (a, a+1)
//   144..151 x_{b-1} x_b for odd b                 (the pairs the columns leave over)
//   152      the constant feature;  153..159 zero
// The 1 + d' + d'^2 layout of the final state is rebuilt from this order in
// write_final_state.
__device__ __forceinline__ uint32_t bmul2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bcast_bf16(uint32_t w, int hi) {
    return __byte_perm(w, w, hi ? 0x3232 : 0x1010);
}

// phi(x) and phi(y) word by word (word w holds features 2w, 2w+1); one copy of
// the code serves both operands, which keeps the kernel's instruction footprint
// small. store(g, wx, wy) receives words 16g..16g+15 of each. Every loop is
// unrolled, so all indices are compile-time constants.
template <typename Store>
__device__ __forceinline__ void emit_phi2(const uint4* xin, uint32_t cx, const uint4* yin, uint32_t cy, Store store) {
    const uint32_t X[8] = {xin[0].x, xin[0].y, xin[0].z, xin[0].w, xin[1].x, xin[1].y, xin[1].z, xin[1].w};
    const uint32_t Y[8] = {yin[0].x, yin[0].y, yin[0].z, yin[0].w, yin[1].x, yin[1].y, yin[1].z, yin[1].w};
    uint32_t bx[16], by[16];
    int n = 0, g = 0;
    auto push = [&](uint32_t wx, uint32_t wy) {
        bx[n] = wx;
        by[n++] = wy;
        if (n == 16) {
            store(g++, bx, by);
            n = 0;
        }
    };
#pragma unroll
    for (int i = 0; i < 8; ++i) push(X[i], Y[i]);                      // x_a
#pragma unroll
    for (int i = 0; i < 8; ++i) {                                       // x_a^2 / sqrt2
        const float x0 = __uint_as_float(X[i] << 16), x1 = __uint_as_float(X[i] & 0xFFFF0000u);
        const float y0 = __uint_as_float(Y[i] << 16), y1 = __uint_as_float(Y[i] & 0xFFFF0000u);
        push(pack_bf16x2((x0 * x0) * kSqrtHalf, (x1 * x1) * kSqrtHalf),
             pack_bf16x2((y0 * y0) * kSqrtHalf, (y1 * y1) * kSqrtHalf));
    }
#pragma unroll
    for (int b = 2; b < DF; ++b) {                                      // column b: pairs (a, a+1), a < 2 floor(b/2)
        const uint32_t xb = bcast_bf16(X[b >> 1], b & 1), yb = bcast_bf16(Y[b >> 1], b & 1);
#pragma unroll
        for (int p = 0; p < b / 2; ++p) push(bmul2(X[p], xb), bmul2(Y[p], yb));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {                                       // x_{b-1} x_b, b = 4k+1 and 4k+3
        push(bmul2(__byte_perm(X[2 * k], X[2 * k + 1], 0x5410), __byte_perm(X[2 * k], X[2 * k + 1], 0x7632)),
             bmul2(__byte_perm(Y[2 * k], Y[2 * k + 1], 0x5410), __byte_perm(Y[2 * k], Y[2 * k + 1], 0x7632)));
    }
    push(cx, cy);                                                       // constant feature, then zero padding
#pragma unroll
    for (int i = 0; i < 3; ++i) push(0u, 0u);
}

// Everything a CTA needs to know about its share of the work.
struct Work {
    size_t bh;               // (b, h)
    int seg, nseg;           // segment index, segments per sequence
    int t_begin, t_end;      // tokens [t_begin, t_end) of the sequence
    int ntiles;              // 128-token tiles of the segment
    bool totals;             // totals pass: state chain only, result to the workspace
    bool has_init;           // main pass, segment > 0: starts from the state the prefix launch wrote
    bool final_state;        // main pass, last segment: writes S and z
    bool packed;             // S and z in the symmetric layout (1 + d' + d'(d'+1)/2 rows)
    float* ws_out;           // totals pass: this part's total
    const float* ws_in;      // main pass: the state entering this segment (rows of KF floats)
    int parts;               // totals per segment (each segment's total is split into parts)
    int sub_tiles;           // tiles per part (the last part of a segment may have fewer)
    const float* gamma;      // coarse decay: gamma of this segment's tiles (index = local tile), or nullptr
    const float* gamma_head; // coarse decay: gamma of the sequence's tiles (index = global tile)
    int c0;                  // global index of this segment's first tile
    int seg_tiles;           // tiles per segment
    const float* ws_base;    // the workspace and its size (floats), for the index checks
    size_t ws_floats;
    unsigned* status;
};

struct Shared {
    uint32_t sbase;
    uint64_t* bars;
    volatile int* abort_flag;
    unsigned* status;
};

// 16 bf16 values (one 16-column TMEM load) as two K-major 16-byte pieces of
// row n of an [S|z] buffer (at byte offset `off`), features 16m..16m+15.
__device__ __forceinline__ void store_sb16(uint32_t sbase, uint32_t off, int n, int m, const float* r) {
    const uint32_t row = sbase + off + (n >> 3) * SB_SBO + (n & 7) * 16;
    st_shared_v4(row + (2 * m) * SB_LBO, pack_bf16x8(r));
    st_shared_v4(row + (2 * m + 1) * SB_LBO, pack_bf16x8(r + 8));
}

// Row stride (floats) of the staged final state: 65 values, 16-byte aligned rows.
constexpr int kStageStride = 68;
static_assert(DS * kStageStride * 4 <= 2 * PK_BYTES, "staged state fits in the phi(K) tiles");

__device__ __forceinline__ unsigned char* smem_generic(uint32_t saddr) {
    extern __shared__ __align__(1024) unsigned char smem[];
    return smem + (saddr - smem_u32(smem));
}

// Whole CTA, after every role has finished: expand the staged folded state
// (stage[f][n], n < 64 for S, n = 64 for z; f in the kernel's feature order) to
// the 1 + d' + d'^2 rows of S and z. Row 1 + d' + a*d' + b takes the folded
// pair (min, max) of (a, b), times 1/sqrt2 off the diagonal (the pair's value
// is split evenly between (a, b) and (b, a)). In the symmetric layout each
// folded pair is one row, unscaled.
__device__ __forceinline__ void write_final_state(const Work& w, uint32_t sbase, int tid, float* S, float* z) {
    const float* stage = reinterpret_cast<const float*>(smem_generic(sbase) + OFF_PK);
    // Kernel feature of folded pair (lo, hi), lo < hi.
    auto pair_source = [](int lo, int hi) {
        if ((hi & 1) && lo == hi - 1) return 144 + (hi - 1) / 2;  // left-over pair of an odd column
        return 32 + 2 * (((hi - 1) * (hi - 1)) / 4) + lo;         // column hi, pairs (a, a+1)
    };
    // Full layout: row r of the 1 + d' + d'^2 rows, with its scale.
    auto source = [&](int r, float& coef) {
        coef = 1.0f;
        if (r == 0) return 152;                                  // constant feature
        if (r <= DF) return r - 1;                               // x_a
        const int p = r - 1 - DF, a = p / DF, b = p % DF;
        if (a == b) return DF + a;                               // x_a^2 / sqrt2
        coef = kSqrtHalf;
        return pair_source(min(a, b), max(a, b));
    };
    // Symmetric layout: row r of the 1 + d' + d'(d'+1)/2 rows (a <= b, a-major),
    // which holds the kernel's folded feature unscaled.
    auto source_packed = [&](int r) {
        if (r == 0) return 152;
        if (r <= DF) return r - 1;
        int a, b;
        packed_pair(r - 1 - DF, DF, a, b);
        return a == b ? DF + a : pair_source(a, b);
    };
    const int D = w.packed ? DS : feature_dim(DF);
    float4* Sd = reinterpret_cast<float4*>(S + w.bh * D * DV);
    const size_t n_heads = gridDim.x / w.nseg;          // extents of S and z for the index checks
    for (int idx = tid; idx < D * (DV / 4); idx += kThreads) {
        const int r = idx / (DV / 4), g = idx % (DV / 4);
        float coef = 1.0f;
        const int f = w.packed ? source_packed(r) : source(r, coef);
        const float4 x = *reinterpret_cast<const float4*>(stage + f * kStageStride + 4 * g);
        if (in_bounds(w.bh * D * DV + 4 * (size_t)idx + 3, n_heads * D * DV, w.status))
            Sd[idx] = make_float4(x.x * coef, x.y * coef, x.z * coef, x.w * coef);
    }
    for (int r = tid; r < D; r += kThreads) {
        float coef = 1.0f;
        const int f = w.packed ? source_packed(r) : source(r, coef);
        if (in_bounds(w.bh * D + r, n_heads * D, w.status)) z[w.bh * D + r] = stage[f * kStageStride + DV] * coef;
    }
}

// Segment start state. Between the totals pass and the main pass a small
// kernel (la_segment_prefix_kernel) turns the totals into running sums: the
// state entering segment s (s >= 1) replaces the first piece of segment s-1 in
// the workspace. The main pass's loader copies that state, row by row, into a
// staging area over the phi(K) tiles, at kInitStride floats per row (padded so
// that the row reads below are free of bank conflicts).
constexpr int kInitStride = KF + 4;
static_assert(NV * kInitStride * 4 <= 2 * PK_BYTES, "segment start state fits in the phi(K) tiles");
constexpr uint32_t kRowBytes = KF * 4;              // one row of a total / start state

// State warps: once the copy has landed, row n of the staged start state into
// the TMEM accumulator (fp32) and into the [S|z] buffer (bf16) for the first
// MMA3; the arrival on INIT also releases the staging area to the producers.
__device__ __forceinline__ void init_state(int n, uint32_t taddr, const Shared& sh) {
    const bool real = n < NV;
    const uint32_t stage = sh.sbase + OFF_PK;
    if (!mbar_wait(&sh.bars[BAR_INITLD], 0, sh.abort_flag, sh.status)) return;
#pragma unroll 1
    for (int m = 0; m < KF / 16; ++m) {
        uint32_t u[16];
        float r[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint4 t = real ? ld_shared_v4(stage + (n * kInitStride + 16 * m + 4 * i) * 4) : make_uint4(0, 0, 0, 0);
            u[4 * i] = t.x;
            u[4 * i + 1] = t.y;
            u[4 * i + 2] = t.z;
            u[4 * i + 3] = t.w;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) r[i] = __uint_as_float(u[i]);
        tmem_st16(taddr + 16 * m, u);
        if (real) store_sb16(sh.sbase, OFF_SB, n, m, r);
    }
    tmem_st_wait();
    fence_proxy_async_smem();
    tc_fence_before();
    mbar_arrive(&sh.bars[BAR_INIT]);
}

// Totals pass with coarse decay: after MMA4 of every tile but the last, scale the
// state by the next tile's gamma in tensor memory and release it (DSF) to the
// next MMA4; the total is then the segment's own decayed state.
__device__ __forceinline__ bool totals_decay_steps(const Work& w, int n, uint32_t taddr, const Shared& sh) {
    for (int c = 0; c + 1 < w.ntiles; ++c) {
        if (!mbar_wait(&sh.bars[BAR_DS], c & 1, sh.abort_flag, sh.status)) return false;
        tc_fence_after();
        const float g = w.gamma[c + 1];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float r[80];
#pragma unroll
            for (int m = 0; m < 5; ++m) tmem_ld16(taddr + 80 * half + 16 * m, r + 16 * m);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 80; ++i) r[i] *= g;
#pragma unroll
            for (int m = 0; m < 5; ++m)
                tmem_st16(taddr + 80 * half + 16 * m, reinterpret_cast<const uint32_t*>(r + 16 * m));
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sh.bars[BAR_DSF]);
    }
    return true;
}

// Totals pass: once the last MMA4 has landed, copy row n of the accumulated
// [S|z]^T (fp32) to this segment's slot in the workspace.
__device__ __forceinline__ void store_total(const Work& w, int n, uint32_t taddr, const Shared& sh) {
    // Without decay the last MMA4 is the only DS commit (phase 0); with decay every
    // tile commits, and the last is phase (ntiles - 1) mod 2.
    const uint32_t parity = w.gamma != nullptr ? (uint32_t)((w.ntiles - 1) & 1) : 0u;
    if (!mbar_wait(&sh.bars[BAR_DS], parity, sh.abort_flag, sh.status)) return;
    tc_fence_after();
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float r[80];
#pragma unroll
        for (int m = 0; m < 5; ++m) tmem_ld16(taddr + 80 * half + 16 * m, r + 16 * m);
        tmem_ld_wait();
        if (n >= NV || !in_bounds((size_t)(w.ws_out - w.ws_base) + (size_t)n * KF + 80 * half + 79, w.ws_floats,
                                  w.status))
            continue;
        float4* dst = reinterpret_cast<float4*>(w.ws_out + (size_t)n * KF + 80 * half);
#pragma unroll
        for (int j = 0; j < 20; ++j) dst[j] = make_float4(r[4 * j], r[4 * j + 1], r[4 * j + 2], r[4 * j + 3]);
    }
}

// One read-out of the state (read-out number r): read the fp32 state row (two
// batches of 80 columns), release it to the next MMA4, and publish it as bf16
// row n of the [S|z] buffer at `sb_off` for the next MMA3 that reads it -- or,
// after the last tile, stage the final state. The buffer is overwritten only
// once the MMA3 that last read it has completed (barrier `free_bar`, phase
// `free_phase`; free_bar < 0: no MMA3 has read it yet). Keeping that order also
// keeps the publish barrier at most one phase ahead of its waiter, since the Y
// issuer waits for the publish before issuing the MMA3 that frees it.
template <bool DECAY>
__device__ __forceinline__ bool state_step(const Work& w, int r, bool last, int free_bar, uint32_t free_phase,
                                           uint32_t sb_off, int pub_bar, int next_tile, int n, uint32_t taddr,
                                           const Shared& sh, float* S, float* z) {
    if (!mbar_wait(&sh.bars[BAR_DS], r & 1, sh.abort_flag, sh.status)) return false;
    tc_fence_after();
    if (!last && free_bar >= 0 && !mbar_wait(&sh.bars[free_bar], free_phase, sh.abort_flag, sh.status)) return false;
    // Coarse decay (CL = 128): tile c+1 reads gamma_{c+1} S_c, and its state update
    // adds to gamma_{c+1} S_c, so the state is scaled in tensor memory before the
    // next MMA4 (which waits for DSF) and published scaled.
    const bool decay = DECAY && !last;
    const float g = decay ? w.gamma[next_tile] : 1.0f;
    float v[80];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
#pragma unroll
        for (int m = 0; m < 5; ++m) tmem_ld16(taddr + 80 * half + 16 * m, v + 16 * m);
        tmem_ld_wait();
        if (decay) {                                     // compiled only into the DECAY kernel
#pragma unroll
            for (int i = 0; i < 80; ++i) v[i] *= g;
#pragma unroll
            for (int m = 0; m < 5; ++m)
                tmem_st16(taddr + 80 * half + 16 * m, reinterpret_cast<const uint32_t*>(v + 16 * m));
            if (half == 1) tmem_st_wait();
        }
        if (half == 1 && !last) {
            tc_fence_before();
            mbar_arrive(&sh.bars[BAR_DSF]);
        }
        if (n >= NV) continue;
        if (!last) {
#pragma unroll
            for (int m = 0; m < 5; ++m) store_sb16(sh.sbase, sb_off, n, 5 * half + m, v + 16 * m);
        } else if (w.final_state && S != nullptr && n <= DV) {
            // Stage the final state for the whole-CTA write-out (write_final_state):
            // stage[f][n], rows of kStageStride floats, over the phi(K) tiles,
            // which nothing reads once the last MMA4 has completed.
            float* stage = reinterpret_cast<float*>(smem_generic(sh.sbase) + OFF_PK);
#pragma unroll
            for (int i = 0; i < 80; ++i) {
                const int f = 80 * half + i;
                if (f < DS) stage[f * kStageStride + n] = v[i];
            }
        }
    }
    if (!last) {
        fence_proxy_async_smem();
        mbar_arrive(&sh.bars[pub_bar]);
    }
    return true;
}

// ------------------------------------------------------------------ producers (warps 0-3)
// Row t of a Q or K stage (32-byte swizzle: the two 16-byte halves of row t
// swap places when bit 2 of t is set).
__device__ __forceinline__ void ld_row32(uint32_t tile, int t, uint4* x) {
    const uint32_t sw = ((t >> 2) & 1) << 4;
    x[0] = ld_shared_v4(tile + t * 32 + sw);
    x[1] = ld_shared_v4(tile + t * 32 + (16 ^ sw));
}

// Thread t = token t of the tile = TMEM lane t. Once the tile's inputs have
// landed (stage s), form phi(k_t) into phi(K) buffer b and phi(q_t) into TMEM.
template <int CL, bool TOT>
__device__ __forceinline__ void producers(const Work& w, const Shared& sh, uint32_t tmem, int warp, int tid) {
    constexpr int KS = ring(CL, TOT);
    const int t = tid;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t cm = (t & 7) * 16;                    // row within a core matrix
    const bool with_q = !w.totals;
    // CL = 64: the first MMA3 pass of a tile reads phi(Q) of rows 0-63 only, the
    // second of rows 64-127 only; the other half's rows hold zeros.
    const bool first_half = CL != 64 || warp < 2;
    const uint32_t zeros[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    // A segment's start state is staged over the phi(K) tiles until INIT.
    if (w.has_init && !mbar_wait(&sh.bars[BAR_INIT], 0, sh.abort_flag, sh.status)) return;
    for (int c = 0; c < w.ntiles; ++c) {
        const int b = c & 1, s = c % KS;
        const bool valid = w.t_begin + c * C + t < w.t_end;
        if (!mbar_wait(&sh.bars[BAR_RF0 + s], (c / KS) & 1, sh.abort_flag, sh.status)) return;
        uint4 kx[2], qx[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
        ld_row32(sh.sbase + stage_k(CL, TOT, s), t, kx);
        if (with_q) ld_row32(sh.sbase + off_q(CL) + s * QK_BYTES, t, qx);
        // phi(K) buffer b is free once MMA4 of tile c-2 has read it; phi(Q) goes
        // to TMEM once the last MMA3 of the previous tile has read it.
        if (c >= 2 && !mbar_wait(&sh.bars[BAR_PKF0 + b], ((c >> 1) - 1) & 1, sh.abort_flag, sh.status)) return;
        const int pqf = CL == 64 ? BAR_PQF_HI : BAR_PQF;
        if (with_q && c >= 1 && !mbar_wait(&sh.bars[pqf], (c - 1) & 1, sh.abort_flag, sh.status)) return;
        tc_fence_after();
        // phi(K) (MN-major: a 16-byte piece is 8 features of token t; tokens past
        // the end contribute nothing) and phi(Q) (TMEM lane t), in one pass.
        const uint32_t pk = sh.sbase + OFF_PK + b * PK_BYTES + cm + (t >> 3) * PK_LBO;
        emit_phi2(kx, valid ? 0x3F80u : 0u, qx, 0x3F80u, [&](int g, const uint32_t* uk, const uint32_t* uq) {
#pragma unroll
            for (int j = 0; j < 4; ++j)
                st_shared_v4(pk + (4 * g + j) * PK_SBO, make_uint4(uk[4 * j], uk[4 * j + 1], uk[4 * j + 2], uk[4 * j + 3]));
            if (with_q) tmem_st16(lane_base + COL_PQ + 16 * g, first_half ? uq : zeros);
        });
        fence_proxy_async_smem();
        mbar_arrive(&sh.bars[BAR_IN0 + b]);
        if (!with_q) continue;
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&sh.bars[BAR_PQIN]);
        if constexpr (CL == 64) {
            // Second pass: once the MMA3 of rows 0-63 has completed, rows 64-127
            // take their phi(Q) and rows 0-63 zeros.
            if (!mbar_wait(&sh.bars[BAR_PQF], c & 1, sh.abort_flag, sh.status)) return;
            tc_fence_after();
            if (first_half) {
#pragma unroll
                for (int g = 0; g < KF / 32; ++g) tmem_st16(lane_base + COL_PQ + 16 * g, zeros);
            } else {
                emit_phi2(qx, 0x3F80u, qx, 0x3F80u, [&](int g, const uint32_t* uq, const uint32_t*) {
                    tmem_st16(lane_base + COL_PQ + 16 * g, uq);
                });
            }
            tmem_st_wait();
            tc_fence_before();
            mbar_arrive(&sh.bars[BAR_PQIN]);
        }
    }
}

// ------------------------------------------------------------------ input loader (warp 14, lane 0)
// Q, K and V of tile c into stage c mod KS (the ring's length) by TMA (Q not in the totals pass),
// once every MMA reading the stage's previous tile has completed. Rows past
// the end of the sequence are zero-filled.
template <int CL, bool TOT>
__device__ __forceinline__ void loader(const Work& w, const Shared& sh, const CUtensorMap* tq, const CUtensorMap* tk,
                                       const CUtensorMap* tv) {
    constexpr int KS = ring(CL, TOT);
    const uint32_t bytes = (w.totals ? 0u : QK_BYTES) + QK_BYTES + V_BYTES;
    if (w.has_init) {                                    // the segment's start state, row n at kInitStride floats
        mbar_expect_tx(&sh.bars[BAR_INITLD], NV * kRowBytes);
        for (int n = 0; n < NV; ++n)
            bulk_load(sh.sbase + OFF_PK + n * kInitStride * 4, w.ws_in + (size_t)n * KF, kRowBytes, &sh.bars[BAR_INITLD]);
    }
    int issued = 0;
    for (int c = 0; c < w.ntiles; ++c, ++issued) {
        const int s = c % KS;
        if (c >= KS && !mbar_wait(&sh.bars[BAR_RE0 + s], ((c / KS) - 1) & 1, sh.abort_flag, sh.status)) break;
        uint64_t* full = &sh.bars[BAR_RF0 + s];
        const int row = w.t_begin + c * C;
        mbar_expect_tx(full, bytes);
        if (!w.totals) tma_load_3d(sh.sbase + off_q(CL) + s * QK_BYTES, tq, full, 0, row, (int)w.bh);
        tma_load_3d(sh.sbase + stage_k(CL, TOT, s), tk, full, 0, row, (int)w.bh);
        tma_load_3d(sh.sbase + stage_v(CL, TOT, s), tv, full, 0, row, (int)w.bh);
    }
    // Nothing may land in shared memory after the CTA exits: wait (bounded) for
    // the last load issued into each stage (already complete unless the CTA is
    // giving up early).
    const uint64_t t0 = global_ns();
    for (int c = max(0, issued - KS); c < issued; ++c)
        while (!mbar_try_wait(&sh.bars[BAR_RF0 + c % KS], (c / KS) & 1) && global_ns() - t0 < kWaitLimitNs) {}
    if (w.has_init)
        while (!mbar_try_wait(&sh.bars[BAR_INITLD], 0) && global_ns() - t0 < kWaitLimitNs) {}
}

// ------------------------------------------------------------------ intra (warps 4-7)
// Thread = token i of the tile = TMEM lane i; WQ = the warp's lane quadrant.
// Row i of A in bf16, by blocks of 32 keys, for intra block number kb. `mode`:
//   0  diagonal block: keys j <= i (blocks above the quadrant's diagonal are
//      zero and are neither loaded nor computed);
//   1  an earlier key tile of the same chunk: every key;
//   2  diagonal block of a tile holding two 64-token chunks: keys j <= i of
//      the query's own chunk (rows 64-127 drop keys 0-63).
// Block kb goes to the 16 TMEM columns col_a(kb) of lane i; the first store
// waits for the previous block's MMA2 to have read them. Arriving on BAR_A
// also releases s to the next block's MMA1.
__device__ __forceinline__ bool intra(const Shared& sh, uint32_t tmem, int wq, int lane, int kb, int mode) {
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    if (!mbar_wait(&sh.bars[BAR_S], kb & 1, sh.abort_flag, sh.status)) return false;
    tc_fence_after();
    const bool full = mode == 1;
    const int first_blk = (mode == 2 && wq >= 2) ? 2 : 0;       // key blocks below this one are another chunk's
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
        uint32_t pw[32];                                         // keys 64h .. 64h+63, two per word
        if ((!full && 2 * h > wq) || 2 * h + 1 < first_blk) {   // every key of this batch is masked
#pragma unroll
            for (int p = 0; p < 32; ++p) pw[p] = 0u;
        } else {
            float sv[64];
#pragma unroll
            for (int m = 0; m < 4; ++m) tmem_ld16(lane_base + COL_S + 64 * h + 16 * m, sv + 16 * m);
            tmem_ld_wait();
#pragma unroll
            for (int p = 0; p < 8; ++p) {
                const int blk = 2 * h + p / 4;                  // key block of this piece (warp-uniform)
                if ((!full && blk > wq) || blk < first_blk) {
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) pw[4 * p + q2] = 0u;
                    continue;
                }
                uint32_t wd[4];
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) {
                    float a0, a1;
                    taylor_pair(sv[8 * p + 2 * q2], sv[8 * p + 2 * q2 + 1], a0, a1);
                    wd[q2] = pack_bf16x2(a0, a1);
                }
                if (!full && blk == wq) {                       // diagonal block: keep keys j <= i
#pragma unroll
                    for (int q2 = 0; q2 < 4; ++q2) {
                        const int kk = (8 * p + 2 * q2) & 31;   // key of the pair's low half, within the block
                        wd[q2] &= (kk <= lane ? 0x0000FFFFu : 0u) | (kk + 1 <= lane ? 0xFFFF0000u : 0u);
                    }
                }
#pragma unroll
                for (int q2 = 0; q2 < 4; ++q2) pw[4 * p + q2] = wd[q2];
            }
        }
        if (h == 0) {
            tc_fence_before();                                  // s has been read
            if (kb > 0 && !mbar_wait(&sh.bars[BAR_AF], (kb - 1) & 1, sh.abort_flag, sh.status)) return false;
            tc_fence_after();
        }
        tmem_st16(lane_base + col_a(2 * h), pw);
        tmem_st16(lane_base + col_a(2 * h + 1), pw + 16);
    }
    tmem_st_wait();
    tc_fence_before();
    mbar_arrive(&sh.bars[BAR_A]);
    return true;
}

// Warps 4-7 of the main pass: for every tile, its intra blocks, then (warps
// 4-6, lanes = value columns) its state read-outs.
template <int CL, bool DECAY>
__device__ __forceinline__ void intra_and_state(const Work& w, const Shared& sh, uint32_t tmem, int wq, int lane,
                                                float* S, float* z) {
    using P = Plan<CL>;
    const int n = wq * 32 + lane;                        // value column == TMEM lane (state role)
    const uint32_t taddr = tmem + (static_cast<uint32_t>(wq * 32) << 16) + COL_ST;
    const bool state = wq < 3;
    if (state && w.has_init) init_state(n, taddr, sh);
    int kb = 0, r = 0;
    for (int c = 0; c < w.ntiles; ++c) {
        const int nb = P::blocks(c);
        for (int j = 0; j < nb; ++j, ++kb) {
            const int mode = CL == 64 ? 2 : (j + 1 < nb ? 1 : 0);
            if (!intra(sh, tmem, wq, lane, kb, mode)) return;
        }
        if (!state) continue;
        const bool last_tile = c + 1 == w.ntiles;
        if constexpr (CL == 64) {
            // After the first 64 tokens: publish into the second buffer, which the
            // previous tile's second MMA3 read.
            if (!state_step<DECAY>(w, r++, false, c >= 1 ? BAR_PQF_HI : -1, (c - 1) & 1, OFF_SB1, BAR_SBR1, c + 1, n,
                                   taddr, sh, S, z))
                return;
            if (!state_step<DECAY>(w, r++, last_tile, BAR_PQF, c & 1, OFF_SB, BAR_SBR, c + 1, n, taddr, sh, S, z))
                return;
        } else {
            if (!P::reads_after(c, w.ntiles)) continue;
            if (!state_step<DECAY>(w, r++, last_tile, BAR_PQF, c & 1, OFF_SB, BAR_SBR, c + 1, n, taddr, sh, S, z))
                return;
        }
    }
}

// ------------------------------------------------------------------ epilogue (warps 8-11)
// Thread = token i = TMEM lane i (wq = the warp's lane quadrant). Y -> y =
// Y[:, :64] / Y[:, 64] in bf16, into the 128-byte swizzled tile b = c & 1 (row
// i, 16-byte piece p at slot p ^ (i & 7)), which the store thread (quadrant 0,
// lane 0) writes out with one TMA store; rows past the end of the sequence are
// clipped by the tensor map.
template <int CL>
__device__ __forceinline__ bool epilogue(const Work& w, const Shared& sh, uint32_t tmem, int c, int wq, int lane,
                                         const CUtensorMap* ty) {
    const int t = wq * 32 + lane;
    const bool store_thread = wq == 0 && lane == 0;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t ys = off_ys(CL);
    const int b = c & 1;
    // At CL = 128 a tile is one intra block whose MMA2 completes Y: its AF commit
    // (phase c) stands for BAR_Y. (The epilogue cannot fall two phases behind:
    // the next tile's MMA2 waits for this epilogue's YF.)
    if (!mbar_wait(&sh.bars[CL == 128 ? BAR_AF : BAR_Y], c & 1, sh.abort_flag, sh.status)) return false;
    tc_fence_after();
    float yv[NV];
#pragma unroll
    for (int m = 0; m < NV / 16; ++m) tmem_ld16(lane_base + COL_Y + 16 * m, yv + 16 * m);
    tmem_ld_wait();
    tc_fence_before();
    mbar_arrive(&sh.bars[BAR_YF]);
    // The store of tile c-1 has been issued; once it has read its tile, that
    // tile is free for tile c+1.
    if (store_thread && c >= 1) {
        bulk_wait_read_all();
        mbar_arrive(&sh.bars[BAR_YSF0 + ((c - 1) & 1)]);
    }
    if (c >= 2 && !mbar_wait(&sh.bars[BAR_YSF0 + b], ((c >> 1) - 1) & 1, sh.abort_flag, sh.status)) return false;
    const float inv = 1.0f / yv[DV];
    const uint32_t row = sh.sbase + ys + b * YS_BYTES + t * 128;
#pragma unroll
    for (int p = 0; p < 8; ++p) {
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) o[e] = yv[8 * p + e] * inv;
        st_shared_v4(row + ((p ^ (t & 7)) << 4), pack_bf16x8(o));
    }
    fence_proxy_async_smem();
    mbar_arrive(&sh.bars[BAR_YSR0 + b]);
    if (store_thread) {
        if (!mbar_wait(&sh.bars[BAR_YSR0 + b], (c >> 1) & 1, sh.abort_flag, sh.status)) return false;
        tma_store_3d(ty, sh.sbase + ys + b * YS_BYTES, 0, w.t_begin + c * C, (int)w.bh);
        bulk_commit();
    }
    return true;
}

// Wait (bounded) for the last commit of an issuer that gave up, so no MMA is in
// flight when the tensor memory is freed.
__device__ __forceinline__ void drain(uint64_t* bar, uint32_t parity) {
    if (bar == nullptr) return;
    const uint64_t t0 = global_ns();
    while (!mbar_try_wait(bar, parity) && global_ns() - t0 < kWaitLimitNs) {}
}

// ------------------------------------------------------------------ Y issuer (warp 13, lane 0)
// Per tile c: MMA3 (phi(Q) against the state at its chunk's start), then for
// each intra block: once its A has been formed (which frees s), MMA1 of the
// next block -- so that the next A is formed while this block's MMA2 and the
// next MMA3 run -- then this block's MMA2. At CL = 256 the even tile's buffer
// is still read by the odd tile's first block, so the Y issuer releases it
// (FREE) only after that block's MMA2. At CL = 64 the tile's second MMA3 (rows
// 64-127, the state after its first chunk) comes after MMA2.
template <int CL>
__device__ __forceinline__ void y_issuer(const Work& w, const Shared& sh, uint32_t tmem) {
    constexpr int KS = stages(CL);
    const uint32_t sb = sh.sbase;
    const uint64_t dsb0 = smem_desc(sb + OFF_SB, SB_LBO, SB_SBO);
    const uint64_t dsb1 = smem_desc(sb + OFF_SB1, SB_LBO, SB_SBO);
    uint64_t* bars = sh.bars;
    uint64_t* last_bar = nullptr;
    uint32_t last_parity = 0;
    int kb = 0;                                          // blocks issued (MMA1 commits on BAR_S)
    auto wait = [&](int bar, uint32_t parity) { return mbar_wait(&bars[bar], parity, sh.abort_flag, sh.status); };
    auto commit = [&](int bar, uint32_t parity) {
        mma_commit(&bars[bar]);
        last_bar = &bars[bar];
        last_parity = parity;
    };
    // s = Q_qt K_kt^T (query tile qt's stage, key tile kt's stage)
    auto mma1 = [&](int qt, int kt) {
        const uint64_t dq = smem_desc_swizzled(sb + off_q(CL) + (qt % KS) * QK_BYTES, 16, QK_SBO, 32);
        const uint64_t dk = smem_desc_swizzled(sb + off_k(CL) + (kt % KS) * QK_BYTES, 16, QK_SBO, 32);
        mma_bf16(tmem + COL_S, dq, dk, ID_QK, 0);
        commit(BAR_S, kb & 1);
        ++kb;
    };
    // Y (+)= phi(Q) [S|z] from the buffer `dsb`
    auto mma3 = [&](uint64_t dsb, bool acc) {
#pragma unroll
        for (int j = 0; j < KF / 16; ++j)
            mma_bf16_ts(tmem + COL_Y, tmem + COL_PQ + 8 * j, dsb + ((j * 2 * SB_LBO) >> 4), ID_INT, (acc || j > 0) ? 1u : 0u);
    };
    // Y (+)= A [V_kt | 1]: key tile kt's V stage with the ones block as its
    // second atom; a K step of 16 tokens is 2048 bytes.
    auto mma2 = [&](int blk, int kt, bool acc) {
        const uint32_t va = sb + off_v(CL) + (kt % KS) * V_BYTES;
        const uint64_t dva = smem_desc_sw128(va, sb + off_ones(CL) - va, 1024);
#pragma unroll
        for (int j = 0; j < C / 16; ++j)
            mma_bf16_ts(tmem + COL_Y, tmem + col_a(j >> 1) + 8 * (j & 1), dva + ((j * 2048) >> 4), ID_AV,
                        (acc || j > 0) ? 1u : 0u);
        commit(BAR_AF, blk & 1);
    };
    // The first block of tile t: against t's own keys, or (CL = 256, t odd) the
    // previous tile's.
    auto first_kt = [](int t) { return (CL == 256 && (t & 1)) ? t - 1 : t; };
    bool ok = wait(BAR_RF0, 0);
    if (ok) {
        tc_fence_after();
        mma1(0, 0);
    }
    for (int c = 0; ok && c < w.ntiles; ++c) {
        const int nb = Plan<CL>::blocks(c);
        const int blk0 = Plan<CL>::blocks_before(c);     // first block of this tile
        if (!wait(BAR_PQIN, (CL == 64 ? 2 * c : c) & 1)) break;
        if (c > 0 && !wait(BAR_YF, (c - 1) & 1)) break;
        // The state MMA3 reads: the state at the tile's chunk start (CL >= 128), or
        // before the tile (CL = 64, rows 0-63). Zero (no MMA3) at a segment's start
        // without an initial state.
        const int chunk_first_tile = CL == 256 ? (c & ~1) : c;
        const bool did3 = chunk_first_tile > 0 || w.has_init;
        if (chunk_first_tile == c) {                     // a new state to wait for
            if (chunk_first_tile > 0) {
                const int pub = CL == 256 ? (c >> 1) - 1 : c - 1;
                if (!wait(BAR_SBR, pub & 1)) break;
            } else if (w.has_init && !wait(BAR_INIT, 0)) {
                break;
            }
        }
        tc_fence_after();
        if (did3) mma3(dsb0, false);
        commit(BAR_PQF, c & 1);
        for (int j = 0; ok && j < nb; ++j) {
            const int blk = blk0 + j;
            if (!wait(BAR_A, blk & 1)) { ok = false; break; }   // A formed: s has been read
            tc_fence_after();
            // MMA1 of the next block: the second block of this tile, or the next tile's first.
            if (j + 1 < nb) {
                mma1(c, c);
            } else if (c + 1 < w.ntiles) {
                if (!wait(BAR_RF0 + (c + 1) % KS, ((c + 1) / KS) & 1)) { ok = false; break; }
                tc_fence_after();
                mma1(c + 1, first_kt(c + 1));
            }
            const int kt = j == 0 ? first_kt(c) : c;
            mma2(blk, kt, did3 || j > 0);
            if (CL == 256 && (c & 1) && j == 0) commit(BAR_RE0 + (c - 1) % KS, ((c - 1) / KS) & 1);
        }
        if (!ok) break;
        // Release this tile's input stage -- at CL = 256 an even tile's only after
        // the odd tile's first block has read it (or when no odd tile follows).
        if (CL != 256 || (c & 1) || c + 1 == w.ntiles) commit(BAR_RE0 + c % KS, (c / KS) & 1);
        if constexpr (CL == 64) {
            // rows 64-127: phi(Q) of the second chunk against the state after the first
            if (!wait(BAR_PQIN, (2 * c + 1) & 1) || !wait(BAR_SBR1, c & 1)) break;
            tc_fence_after();
            mma3(dsb1, true);
            commit(BAR_PQF_HI, c & 1);
        }
        if (CL != 128) commit(BAR_Y, c & 1);         // CL = 128: the epilogue waits for AF
    }
    if (*sh.abort_flag) drain(last_bar, last_parity);
}

// ------------------------------------------------------------------ state issuer (warp 12, lane 0)
// MMA4 of every tile, in Plan::kSteps steps of 128 / kSteps tokens; a DS commit
// after every step that a read-out follows, and before the next step the wait
// for that read-out (DSF).
template <int CL, bool TOT>
__device__ __forceinline__ void state_issuer(const Work& w, const Shared& sh, uint32_t tmem) {
    using P = Plan<CL>;
    constexpr int kSteps = P::kSteps;
    constexpr int kJ = C / 16 / kSteps;                  // K steps of 16 tokens per MMA4 step
    constexpr int KS = ring(CL, TOT);
    const uint32_t sb = sh.sbase;
    const uint64_t dpk0 = smem_desc(sb + OFF_PK, PK_LBO, PK_SBO);    // phi(K): N = feature, MN-major
    uint64_t* bars = sh.bars;
    uint64_t* last_bar = nullptr;
    uint32_t last_parity = 0;
    auto wait = [&](int bar, uint32_t parity) { return mbar_wait(&bars[bar], parity, sh.abort_flag, sh.status); };
    // Read-outs: every step in the main pass (at CL = 256 after odd tiles and
    // the last); in the totals pass only after the last tile, or every tile
    // with decay (the state is rescaled per tile).
    const bool decay_totals = w.totals && w.gamma != nullptr;
    int r = 0;                                           // read-outs committed so far
    bool pending = false;                                // a read-out follows the previous step
    bool ok = !w.has_init || wait(BAR_INIT, 0);
    for (int c = 0; ok && c < w.ntiles; ++c) {
        const int b = c & 1, s = c % KS;
        if (!wait(BAR_RF0 + s, (c / KS) & 1) || !wait(BAR_IN0 + b, (c >> 1) & 1)) break;
        // [V|1]^T as the A operand (M = column: V's atom, then the ones block; K = token)
        const uint32_t va = sb + stage_v(CL, TOT, s);
        const uint64_t dva = smem_desc_sw128(va, sb + off_ones(CL) - va, 1024);
        for (int h = 0; h < kSteps; ++h) {
            if (pending && !wait(BAR_DSF, (r - 1) & 1)) { ok = false; break; }
            tc_fence_after();
            const uint64_t dpk = dpk0 + ((b * PK_BYTES) >> 4);
#pragma unroll
            for (int jj = 0; jj < kJ; ++jj) {
                const int j = h * kJ + jj;
                mma_bf16(tmem + COL_ST, dva + ((j * 2048) >> 4), dpk + ((j * 2 * PK_LBO) >> 4), ID_UPD,
                         (c > 0 || j > 0 || w.has_init) ? 1u : 0u);
            }
            if (h + 1 == kSteps) {
                mma_commit(&bars[BAR_PKF0 + b]);
                mma_commit(&bars[BAR_RE0 + s]);
                last_bar = &bars[BAR_RE0 + s];
                last_parity = (c / KS) & 1;
            }
            const bool last = c + 1 == w.ntiles && h + 1 == kSteps;
            bool readout;
            if (w.totals) readout = last || decay_totals;
            else readout = CL == 64 || P::reads_after(c, w.ntiles);
            if (readout) {
                mma_commit(&bars[BAR_DS]);
                last_bar = &bars[BAR_DS];
                last_parity = (uint32_t)(w.totals && !decay_totals ? 0 : r & 1);
                ++r;
            }
            pending = readout && !last && (!w.totals || decay_totals);
        }
    }
    if (*sh.abort_flag) drain(last_bar, last_parity);
}

// TOT false: main pass over every segment; TOT true: totals pass over segments
// 0..nseg-2, each split into `parts` pieces of at most sub_tiles = ceil(seg_tiles /
// parts) tiles (only the state chain and its read-out are compiled in).
// SEG: compiled for more than one segment per sequence (a segment may start from
// a state); without it, every CTA starts from zero and none of that code exists.
template <int CL, bool DECAY, bool SEG, bool TOT>
__global__ void __launch_bounds__(kThreads, 1)
la_prefill_tc_kernel(const __grid_constant__ CUtensorMap ty, const __grid_constant__ CUtensorMap tq,
                     const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                     float* __restrict__ S, float* __restrict__ z, int N, int nseg, int seg_tiles, int parts,
                     int packed, float* __restrict__ ws, const float* __restrict__ gamma, unsigned* status,
                     unsigned debug) {
    static_assert(!DECAY || CL == 128, "coarse decay is per 128-token tile, with 128-token chunks");
    static_assert(!TOT || SEG, "the totals pass exists only with segments");
    extern __shared__ __align__(1024) unsigned char smem[];
    constexpr uint32_t kOffBar = off_bar(CL);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
    uint32_t* tmem_base_slot = reinterpret_cast<uint32_t*>(smem + kOffBar + 8 * NUM_BARS);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffBar + 8 * NUM_BARS + 4);
    const Shared sh{smem_u32(smem), bars, abort_flag, status};

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;

    if (warp == 14 && lane == 0) {                       // the loader's maps (and the y stores')
        prefetch_tensormap(&tk);
        prefetch_tensormap(&tv);
        if (!TOT) {
            prefetch_tensormap(&tq);
            prefetch_tensormap(&ty);
        }
    }

    Work w;
    w.totals = TOT;
    w.parts = parts;
    w.sub_tiles = (seg_tiles + parts - 1) / parts;
    const int per_head = w.totals ? (nseg - 1) * parts : nseg;
    w.bh = blockIdx.x / per_head;
    const int j = blockIdx.x % per_head;
    w.seg = w.totals ? j / parts : j;
    w.nseg = nseg;
    if (w.totals) {                                      // part j % parts of segment seg
        const int p = j % parts;
        w.t_begin = (w.seg * seg_tiles + p * w.sub_tiles) * C;
        w.t_end = min(N, (w.seg * seg_tiles + min((p + 1) * w.sub_tiles, seg_tiles)) * C);
    } else {
        w.t_begin = w.seg * seg_tiles * C;
        w.t_end = min(N, w.t_begin + seg_tiles * C);
    }
    w.ntiles = (w.t_end - w.t_begin + C - 1) / C;
    w.has_init = SEG && !w.totals && w.seg > 0;
    w.final_state = !w.totals && w.seg == nseg - 1;
    w.packed = packed != 0;
    w.ws_out = w.totals ? ws + (w.bh * (nseg - 1) * parts + j) * kTotalFloats : nullptr;
    w.ws_in = w.has_init ? ws + (w.bh * (nseg - 1) * parts + (size_t)(w.seg - 1) * parts) * kTotalFloats : nullptr;
    w.c0 = w.t_begin / C;
    w.seg_tiles = seg_tiles;
    w.ws_base = ws;
    w.ws_floats = (size_t)(gridDim.x / per_head) * (nseg - 1) * parts * kTotalFloats;
    w.status = status;
    w.gamma_head = gamma != nullptr ? gamma + w.bh * (size_t)((N + C - 1) / C) : nullptr;
    w.gamma = gamma != nullptr ? w.gamma_head + w.c0 : nullptr;

    if (tid == 0) {
        for (int i = 0; i < NUM_BARS; ++i) {
            uint32_t count = 1;
            if (i == BAR_IN0 || i == BAR_IN1 || i == BAR_PQIN || i == BAR_A || i == BAR_YF || i == BAR_YSR0 ||
                i == BAR_YSR1)
                count = 128;                                 // one warpgroup
            if (i == BAR_DSF || i == BAR_SBR || i == BAR_SBR1 || i == BAR_INIT) count = kStateLanes;
            if (i >= BAR_RE0 && i <= BAR_RE3 && !w.totals) count = 2;   // both issuers read an input stage
            mbar_init(&bars[i], count);
        }
        *abort_flag = 0;
        mbar_fence_init();
    }
    if (warp == 13) tmem_alloc(tmem_base_slot, TMEM_COLS);
    {
        // The ones block: row t (token) holds bf16 1.0 in column 64, i.e. in its
        // 16-byte piece 0, which the 128-byte swizzle stores at slot (t mod 8).
        const uint32_t ones = sh.sbase + off_ones(CL);
        for (int i = tid; i < C * 8; i += kThreads) {
            const int row = i >> 3, slot = i & 7;
            st_shared_v4(ones + row * 128 + slot * 16, make_uint4(slot == (row & 7) ? 0x3F80u : 0u, 0u, 0u, 0u));
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_base_slot;
    grid_dependency_wait();                              // inputs and workspace may come from the previous kernel

    const bool skip_mma = (debug & DEBUG_SKIP_MMA) != 0;   // testing: issue nothing, every waiter times out

    if (warp < 4) {
        producers<CL, TOT>(w, sh, tmem, warp, tid);
    } else if (warp < 8) {
        const int wq = warp & 3;
        if (w.totals) {
            const int n = wq * 32 + lane;
            const uint32_t taddr = tmem + (static_cast<uint32_t>(wq * 32) << 16) + COL_ST;
            if (wq < 3 && (w.gamma == nullptr || totals_decay_steps(w, n, taddr, sh))) store_total(w, n, taddr, sh);
        } else {
            intra_and_state<CL, DECAY>(w, sh, tmem, wq, lane, S, z);
        }
    } else if (warp < 12) {
        if (!w.totals) {
            const int wq = warp & 3;
            for (int c = 0; c < w.ntiles; ++c)
                if (!epilogue<CL>(w, sh, tmem, c, wq, lane, &ty)) break;
            if (wq == 0 && lane == 0) bulk_wait_all();      // the y stores have completed
        }
    } else if (warp == 12) {
        if (lane == 0 && !skip_mma) state_issuer<CL, TOT>(w, sh, tmem);
    } else if (warp == 13) {
        if (lane == 0 && !w.totals && !skip_mma) y_issuer<CL>(w, sh, tmem);
    } else {
        if (lane == 0) loader<CL, TOT>(w, sh, &tq, &tk, &tv);
    }

    tc_fence_before();
    __syncthreads();
    if (w.final_state && S != nullptr && !*abort_flag) write_final_state(w, sh.sbase, tid, S, z);
    if (warp == 13) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc(tmem, TMEM_COLS);
    }
}

// Running sums of the segment totals, in place. Thread = one float4 column of a
// total (16 rows x 4 features of the KF-wide rows), blockIdx.y = the sequence.
// Walking the pieces of segments 0..nseg-2 in order, the state entering
// segment s+1 replaces the first piece of segment s, which this thread has
// read by then (each thread touches only its own column). With coarse decay
// (DECAY) a piece's total counts with the product of gamma over its own tiles
// on the state before it, and the state handed to segment s+1 takes the gamma
// of that segment's first tile.
template <bool DECAY>
__global__ void __launch_bounds__(256)
la_segment_prefix_kernel(float* __restrict__ ws, int nseg, int parts, int seg_tiles, const float* __restrict__ gamma,
                         int seq_tiles) {
    grid_dependency_wait();                              // the totals pass has written the pieces
    constexpr int kCols = (int)(kTotalFloats / 4);
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= kCols) return;
    float4* base = reinterpret_cast<float4*>(ws) + (size_t)blockIdx.y * (nseg - 1) * parts * kCols;
    const float* g = DECAY ? gamma + (size_t)blockIdx.y * seq_tiles : nullptr;
    const int sub = (seg_tiles + parts - 1) / parts;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int sg = 0; sg + 1 < nseg; ++sg) {
        for (int p = 0; p < parts; ++p) {
            const float4 t = base[(size_t)(sg * parts + p) * kCols + i];
            if constexpr (DECAY) {
                float d = 1.0f;
                const int c_hi = sg * seg_tiles + min((p + 1) * sub, seg_tiles);
                for (int c = sg * seg_tiles + p * sub; c < c_hi; ++c) d *= g[c];
                acc = make_float4(acc.x * d, acc.y * d, acc.z * d, acc.w * d);
            }
            acc = make_float4(acc.x + t.x, acc.y + t.y, acc.z + t.z, acc.w + t.w);
        }
        const float g0 = DECAY ? g[(sg + 1) * seg_tiles] : 1.0f;
        base[(size_t)(sg * parts) * kCols + i] = make_float4(acc.x * g0, acc.y * g0, acc.z * g0, acc.w * g0);
    }
}

// Segments per sequence: enough CTAs to cover the SMs once, whole chunks each
// (tiles_per_chunk tiles of 128 tokens per chunk).
void plan_segments(int BH, int N, int num_sms, int tiles_per_chunk, int* nseg, int* seg_tiles) {
    const int chunk_tokens = C * tiles_per_chunk;
    const int nchunks = (N + chunk_tokens - 1) / chunk_tokens;
    int n = 1;
    if (BH < num_sms) n = std::min(nchunks, std::max(1, num_sms / BH));
    const int per = (nchunks + n - 1) / n;
    *seg_tiles = per * tiles_per_chunk;
    *nseg = (nchunks + per - 1) / per;
}

int tiles_per_chunk(int chunk) { return chunk > C ? chunk / C : 1; }

// Pieces per segment total in the totals pass: the most even use of the SMs.
// A total splits into `parts` pieces of consecutive tiles (each its own CTA);
// the pass takes about ceil(CTAs / SMs) rounds of (tiles per piece + ~2 tiles of
// start-up and store). Only splits whose totals fit `ws_cap` bytes, and whose
// last piece is not empty, are considered.
int plan_parts(int BH, int nseg, int seg_tiles, int num_sms, size_t ws_cap) {
    if (nseg <= 1) return 1;
    const long long units = (long long)BH * (nseg - 1);
    int best = 1;
    double best_cost = 1e30;
    for (int p = 1; p <= std::min(seg_tiles, 16); ++p) {
        const int sub = (seg_tiles + p - 1) / p;
        if ((p - 1) * sub >= seg_tiles) continue;
        if ((size_t)units * p * kTotalFloats * sizeof(float) > ws_cap) break;
        const long long waves = (units * p + num_sms - 1) / num_sms;
        const double cost = (double)waves * (sub + 2.0);
        if (cost < best_cost - 1e-9) {
            best_cost = cost;
            best = p;
        }
    }
    return best;
}

template <int CL>
cudaError_t launch_cl(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    const int BH = a.B * a.H;
    int nseg, seg_tiles;
    plan_segments(BH, a.N, num_sms, tiles_per_chunk(CL), &nseg, &seg_tiles);
    auto kern = nseg > 1 ? la_prefill_tc_kernel<CL, false, true, false> : la_prefill_tc_kernel<CL, false, false, false>;
    auto ktot = la_prefill_tc_kernel<CL, false, true, true>;
    if constexpr (CL == 128)
        if (a.gamma != nullptr) {
            kern = nseg > 1 ? la_prefill_tc_kernel<128, true, true, false> : la_prefill_tc_kernel<128, true, false, false>;
            ktot = la_prefill_tc_kernel<128, true, true, true>;
        }
    constexpr uint32_t kSmem = smem_bytes(CL);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e == cudaSuccess && nseg > 1)
        e = cudaFuncSetAttribute(ktot, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
    if (e != cudaSuccess) return e;
    float* ws = static_cast<float*>(a.workspace);
    // Split the totals as finely as helps and as the given workspace holds (the
    // workspace query sizes it for the best split; a smaller one, as the
    // allocation-free entry point has, takes fewer pieces).
    const int parts = plan_parts(BH, nseg, seg_tiles, num_sms, a.ws_bytes);
    if (nseg > 1 && (ws == nullptr || a.ws_bytes < (size_t)BH * (nseg - 1) * parts * kTotalFloats * sizeof(float)))
        return cudaErrorInvalidValue;                    // the segment totals need their workspace
    CUtensorMap ty, tq, tk, tv;
    if (!make_tmap_bf16_3d(&ty, a.y, DV, a.N, BH, DV, C) ||
        !make_tmap_bf16_3d_swizzle(&tq, a.q, DF, a.N, BH, DF, C, 32) ||
        !make_tmap_bf16_3d_swizzle(&tk, a.k, DF, a.N, BH, DF, C, 32) ||
        !make_tmap_bf16_3d_swizzle(&tv, a.v, DV, a.N, BH, DV, C, 128))
        return cudaErrorInvalidValue;
    if (nseg > 1) {
        e = launch_pdl(ktot, dim3(BH * (nseg - 1) * parts), dim3(kThreads), kSmem, stream, ty, tq, tk, tv, a.S,
                       a.z, a.N, nseg, seg_tiles, parts, a.packed ? 1 : 0, ws, a.gamma, a.status, a.debug);
        if (e != cudaSuccess) return e;
        const dim3 pgrid((unsigned)((kTotalFloats / 4 + 255) / 256), (unsigned)BH);
        const int seq_tiles = (a.N + C - 1) / C;
        e = a.gamma != nullptr
                ? launch_pdl(la_segment_prefix_kernel<true>, pgrid, dim3(256), 0, stream, ws, nseg, parts, seg_tiles,
                             a.gamma, seq_tiles)
                : launch_pdl(la_segment_prefix_kernel<false>, pgrid, dim3(256), 0, stream, ws, nseg, parts, seg_tiles,
                             a.gamma, seq_tiles);
        if (e != cudaSuccess) return e;
    }
    return launch_pdl(kern, dim3(BH * nseg), dim3(kThreads), kSmem, stream, ty, tq, tk, tv, a.S,
                      a.z, a.N, nseg, seg_tiles, parts, a.packed ? 1 : 0, ws, a.gamma, a.status, a.debug);
}

}  // namespace

bool la_prefill_tc_supported(int d_feat, int d_v, int chunk) {
    return d_feat == DF && d_v == DV && (chunk == 64 || chunk == 128 || chunk == 256);
}

size_t la_prefill_tc_workspace(int B, int H, int N, int d_feat, int d_v, int chunk, int num_sms) {
    if (!la_prefill_tc_supported(d_feat, d_v, chunk)) return 0;
    int nseg, seg_tiles;
    plan_segments(B * H, N, num_sms, tiles_per_chunk(chunk), &nseg, &seg_tiles);
    const int parts = plan_parts(B * H, nseg, seg_tiles, num_sms, ~(size_t)0);
    return (size_t)B * H * (nseg - 1) * parts * kTotalFloats * sizeof(float);
}

size_t la_prefill_tc_workspace_min(int B, int H, int N, int d_feat, int d_v, int chunk, int num_sms) {
    if (!la_prefill_tc_supported(d_feat, d_v, chunk)) return 0;
    int nseg, seg_tiles;
    plan_segments(B * H, N, num_sms, tiles_per_chunk(chunk), &nseg, &seg_tiles);
    return (size_t)B * H * (nseg - 1) * kTotalFloats * sizeof(float);
}

cudaError_t launch_la_prefill_tc(const LaPrefillArgs& a, int num_sms, cudaStream_t stream) {
    if (!la_prefill_tc_supported(a.d_feat, a.d_v, a.chunk) || !a.bf16) return cudaErrorInvalidValue;
    if (a.gamma != nullptr && a.chunk != 128) return cudaErrorInvalidValue;   // decay tiles are the 128-token chunks
    switch (a.chunk) {
        case 64: return launch_cl<64>(a, num_sms, stream);
        case 256: return launch_cl<256>(a, num_sms, stream);
        default: return launch_cl<128>(a, num_sms, stream);
    }
}

}  // namespace based

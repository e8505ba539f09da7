// Recurrent (next-token) step of causal Taylor linear attention.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), §2 "Efficient attentions" (recurrent generation at O(1)
// per token) and App. B "Next Token Prediction" (KV-state update kernel):
//     S += phi(k) v^T,  z += phi(k),  y = phi(q)^T S / phi(q)^T z.
//
// The step is bound by HBM: each (b, h) reads and writes its fp32 state once
// (D x dv + D floats, 70 KB at d' = 16, dv = 64) while doing ~0.5 flop per byte.
// The same kernel serves the symmetric layout (1 + d' + d'(d'+1)/2 rows: 39 KB
// at d' = 16), whose rows (a, b), a <= b, hold x_a x_b unscaled off the
// diagonal; each CTA tabulates the pairs of its rows once.
//
// Work split: a head's D feature rows are cut into P contiguous row ranges,
// one CTA each, and the P CTAs of a head form one thread-block cluster
// (P in {1, 2, 4, 8}, chosen so the grid covers every SM about twice even at
// batch 1). Rows of S and z are disjoint between the CTAs, so the in-place
// update never races; each CTA produces a partial numerator phi(q)_rows . S_rows
// (dv values) and a partial denominator phi(q)_rows . z_rows, and rank 0 of the
// cluster sums the P partials through distributed shared memory and writes y.
//
// Streaming: a thread owns one 16-byte column group of every (kThreads / G)-th
// row of its range. It issues the loads of a batch of kBatch rows before it
// needs any of them, and the first batch is in flight before q, k and v have
// even arrived, so the load latency overlaps the feature-map setup. phi(q) and
// phi(k) are formed per row from q and k held in shared memory (two multiplies)
// and never reach HBM.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace based {
namespace {

namespace cg = cooperative_groups;

constexpr int kThreads = 256;
constexpr int kBatch = 8;        // rows in flight per thread
constexpr int kMaxRanks = 8;     // portable cluster size

template <int DF>
__device__ __forceinline__ float phi_entry(const float* x, int f) {
    if (f == 0) return 1.0f;
    if (f <= DF) return x[f - 1];
    const int p = f - 1 - DF;
    return (x[p / DF] * x[p % DF]) * kSqrtHalf;
}

// Feature f of the symmetric layout; `pair` = (a << 8) | b of its pair (a <= b).
template <int DF>
__device__ __forceinline__ float phi_entry_packed(const float* x, int f, unsigned pair) {
    if (f == 0) return 1.0f;
    if (f <= DF) return x[f - 1];
    const int a = pair >> 8, b = pair & 0xFF;
    const float p = x[a] * x[b];
    return a == b ? p * kSqrtHalf : p;
}

__device__ __forceinline__ void fma4(float4& acc, float s, const float4& x) {
    acc.x = fmaf(s, x.x, acc.x);
    acc.y = fmaf(s, x.y, acc.y);
    acc.z = fmaf(s, x.z, acc.z);
    acc.w = fmaf(s, x.w, acc.w);
}

template <typename T, int DF, int DV, bool PACKED>
__global__ void __launch_bounds__(kThreads)
la_decode_kernel(float* __restrict__ S, float* __restrict__ z, const T* __restrict__ q,
                 const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ y,
                 const float* __restrict__ gamma, int P, unsigned* status) {
    constexpr int D = PACKED ? sym_feature_dim(DF) : feature_dim(DF);
    constexpr int G = DV / 4;              // float4 column groups per row
    constexpr int RPS = kThreads / G;      // rows per sweep of the CTA
    constexpr int NW = kThreads / 32;
    static_assert(kThreads % G == 0 && G <= 32 && 32 % G == 0, "thread layout");

    __shared__ float s_x[2][DF];
    __shared__ float s_v[DV];
    __shared__ float4 s_red[NW][G];
    __shared__ float s_dred[NW];
    __shared__ float s_out[DV + 1];        // this CTA's partial numerator and denominator
    __shared__ unsigned short s_pair[PACKED ? 2 * kThreads : 1];   // pair (a, b) of this CTA's rows

    const int tid = threadIdx.x;
    const int rank = (int)(blockIdx.x % (unsigned)P);
    const size_t bh = blockIdx.x / (unsigned)P;
    const int f0 = (rank * D) / P;
    const int f1 = ((rank + 1) * D) / P;
    const int g = tid % G;
    const int r_thr = tid / G;

    float* Sp = S + (bh * D) * (size_t)DV + 4 * g;
    const size_t n_heads = gridDim.x / (unsigned)P;       // extents of S, z and y for the index checks
    grid_dependency_wait();

    // First batch of state rows: in flight before anything else.
    float4 buf[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
        const int f = f0 + r_thr + u * RPS;
        if (f < f1) buf[u] = *reinterpret_cast<const float4*>(Sp + (size_t)f * DV);
    }

    // Decay of the state before this token (1 without decay): S <- gamma S, z <- gamma z.
    const float gdec = gamma != nullptr ? gamma[bh] : 1.0f;

    // This thread's z rows (at most two: a CTA holds at most 2 * kThreads rows).
    float* zbh = z + bh * D;
    float zr[2];
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int f = f0 + tid + i * kThreads;
        if (f < f1) zr[i] = zbh[f];
    }

    if (tid < DF) {
        s_x[0][tid] = to_f32(q[bh * DF + tid]);
        s_x[1][tid] = to_f32(k[bh * DF + tid]);
    }
    if (tid < DV) s_v[tid] = to_f32(v[bh * DV + tid]);
    if constexpr (PACKED) {
        for (int j = tid; j < f1 - f0; j += kThreads) {
            int a = 0, b = 0;
            if (f0 + j > DF) packed_pair(f0 + j - 1 - DF, DF, a, b);
            s_pair[j] = (unsigned short)((a << 8) | b);
        }
    }
    __syncthreads();
    auto phi = [&](const float* x, int f) {
        if constexpr (PACKED) return phi_entry_packed<DF>(x, f, s_pair[f - f0]);
        else return phi_entry<DF>(x, f);
    };

    // Denominator part over this CTA's rows; z updated in place.
    float dpart = 0.f;
#pragma unroll
    for (int i = 0; i < 2; ++i) {
        const int f = f0 + tid + i * kThreads;
        if (f < f1) {
            const float zn = fmaf(gdec, zr[i], phi(s_x[1], f));
            if (in_bounds(bh * D + f, n_heads * D, status)) zbh[f] = zn;
            dpart = fmaf(phi(s_x[0], f), zn, dpart);
        }
    }

    const float4 vv = make_float4(s_v[4 * g], s_v[4 * g + 1], s_v[4 * g + 2], s_v[4 * g + 3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int base = f0 + r_thr;; base += kBatch * RPS) {
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int f = base + u * RPS;
            if (f < f1) {
                float4 s = make_float4(gdec * buf[u].x, gdec * buf[u].y, gdec * buf[u].z, gdec * buf[u].w);
                fma4(s, phi(s_x[1], f), vv);
                if (in_bounds((bh * D + f) * DV + 4 * g + 3, n_heads * D * DV, status))
                    *reinterpret_cast<float4*>(Sp + (size_t)f * DV) = s;
                fma4(acc, phi(s_x[0], f), s);
            }
        }
        const int next = base + kBatch * RPS;
        if (next >= f1) break;
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int f = next + u * RPS;
            if (f < f1) buf[u] = *reinterpret_cast<const float4*>(Sp + (size_t)f * DV);
        }
    }

    // CTA reduction: lanes of a warp that share a column group, then warps.
    const int warp = tid >> 5, lane = tid & 31;
#pragma unroll
    for (int o = G; o < 32; o <<= 1) {
        acc.x += __shfl_xor_sync(0xffffffffu, acc.x, o);
        acc.y += __shfl_xor_sync(0xffffffffu, acc.y, o);
        acc.z += __shfl_xor_sync(0xffffffffu, acc.z, o);
        acc.w += __shfl_xor_sync(0xffffffffu, acc.w, o);
    }
    if (lane < G) s_red[warp][lane] = acc;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dpart += __shfl_xor_sync(0xffffffffu, dpart, o);
    if (lane == 0) s_dred[warp] = dpart;
    __syncthreads();
    if (tid < DV) {
        float num = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) num += reinterpret_cast<const float*>(&s_red[w][tid >> 2])[tid & 3];
        s_out[tid] = num;
    } else if (tid == DV) {
        float den = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) den += s_dred[w];
        s_out[DV] = den;
    }

    // Cluster reduction through distributed shared memory; rank 0 writes y.
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();
    if (rank == 0 && tid < DV) {
        float num = 0.f, den = 0.f;
        for (int r = 0; r < P; ++r) {
            const float* o = cluster.map_shared_rank(s_out, r);
            num += o[tid];
            den += o[DV];
        }
        if (in_bounds(bh * DV + tid, n_heads * DV, status)) y[bh * DV + tid] = from_f32<T>(num / den);
    }
    cluster.sync();   // keep every rank's shared memory alive until rank 0 has read it
}

// Ranks per head: doubled while the grid is below twice the SM count, at least
// 16 rows per CTA, a power of two up to the portable cluster size. At H=16,
// d'=16, dv=64 that is 4 ranks at batch 8 and 2 at batch 16. A four-fold
// cover (8 and 4 ranks) was ~15 % slower with L2 flushed between calls; in the
// bench step's graph, stopping below twice the SMs (2 and 1 ranks) was 5-6 %
// slower.
int ranks_per_head(int BH, int D, int num_sms) {
    int P = 1;
    while (P < kMaxRanks && (long long)BH * P < 2LL * num_sms && D / (2 * P) >= 16) P *= 2;
    while ((D + P - 1) / P > 2 * kThreads) P *= 2;    // z rows per thread: at most two
    return P;
}

template <typename T, int DF, int DV, bool PACKED>
cudaError_t launch_typed(float* S, float* z, const void* q, const void* k, const void* v, void* y,
                         const float* gamma, int BH, int num_sms, unsigned* status, cudaStream_t stream) {
    const int P = ranks_per_head(BH, PACKED ? sym_feature_dim(DF) : feature_dim(DF), num_sms);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)BH * P);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = P;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    // Programmatic dependent launch: the CTAs are scheduled while the previous
    // kernel drains and wait (griddepcontrol) before reading anything.
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, la_decode_kernel<T, DF, DV, PACKED>, S, z, static_cast<const T*>(q),
                              static_cast<const T*>(k), static_cast<const T*>(v), static_cast<T*>(y), gamma, P,
                              status);
}

template <typename T, bool PACKED>
cudaError_t dispatch(float* S, float* z, const void* q, const void* k, const void* v, void* y,
                     const float* gamma, int BH, int d_feat, int d_v, int num_sms, unsigned* status,
                     cudaStream_t stream) {
    if (d_feat == 16 && d_v == 64)
        return launch_typed<T, 16, 64, PACKED>(S, z, q, k, v, y, gamma, BH, num_sms, status, stream);
    if (d_feat == 16 && d_v == 128)
        return launch_typed<T, 16, 128, PACKED>(S, z, q, k, v, y, gamma, BH, num_sms, status, stream);
    if (d_feat == 32 && d_v == 64)
        return launch_typed<T, 32, 64, PACKED>(S, z, q, k, v, y, gamma, BH, num_sms, status, stream);
    if (d_feat == 32 && d_v == 128)
        return launch_typed<T, 32, 128, PACKED>(S, z, q, k, v, y, gamma, BH, num_sms, status, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_la_decode(float* S, float* z, const void* q, const void* k, const void* v,
                             void* y, const float* gamma, int B, int H, int d_feat, int d_v, bool bf16, bool packed,
                             int num_sms, unsigned* status, cudaStream_t stream) {
    const int BH = B * H;
    if (packed)
        return bf16 ? dispatch<__nv_bfloat16, true>(S, z, q, k, v, y, gamma, BH, d_feat, d_v, num_sms, status, stream)
                    : dispatch<float, true>(S, z, q, k, v, y, gamma, BH, d_feat, d_v, num_sms, status, stream);
    return bf16 ? dispatch<__nv_bfloat16, false>(S, z, q, k, v, y, gamma, BH, d_feat, d_v, num_sms, status, stream)
                : dispatch<float, false>(S, z, q, k, v, y, gamma, BH, d_feat, d_v, num_sms, status, stream);
}

}  // namespace based

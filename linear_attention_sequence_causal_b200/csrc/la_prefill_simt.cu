// Chunked causal Taylor linear attention on the CUDA cores, fp32 arithmetic.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), App. B "Forward / Generation Prefill": the output of a
// tile of C tokens is an on-diagonal part (the causal quadratic form inside the
// tile) plus an off-diagonal part read from the cumulative state of all earlier
// tiles; "Gated Slot Attention" App. A.1 calls these the intra- and inter-chunk
// terms. For chunk c:
//     A   = (1 + Q_c K_c^T + (Q_c K_c^T)^2 / 2) masked to j <= i
//     y_c = (A V_c + phi(Q_c) S) / (rowsum A + phi(Q_c) z)
//     S  += phi(K_c)^T V_c,   z += colsum phi(K_c)
// (with coarse decay, S and z are first scaled by gamma where a 128-token tile
// begins).
//
// This is the fp32 path (fp32 inputs, and any (d', dv) without a tensor-core
// kernel). Each CTA owns one (b, h) and a 16-column slice of dv, keeps its slice
// of S and all of z in shared memory for the whole sequence and recomputes the
// (cheap) intra-chunk weights and denominator itself, so CTAs never exchange
// data. phi is formed in shared memory only.
//
// State inside the kernel uses the symmetric fold of the order-2 block:
// (q.k)^2/2 = sum_a (q_a^2/sqrt2)(k_a^2/sqrt2) + sum_{a<b} (q_a q_b)(k_a k_b),
// i.e. 1 + d' + d'(d'+1)/2 distinct features instead of 1 + d' + d'^2. The final
// state is written out in the full layout: S[1+d'+a*d'+b] = S[1+d'+b*d'+a] is
// the folded entry scaled by 1/sqrt2 when a != b, and the folded entry itself
// when a == b -- or, for the packed entry points, as it is (the fold is the
// symmetric layout).
#include "common.cuh"
#include "kernels.h"

namespace based {
namespace {

constexpr int kThreads = 256;
constexpr int kCW = 16;   // dv columns per CTA

// Index of the folded pair (a <= b) among the order-2 features.
__host__ __device__ constexpr int pair_index(int a, int b, int DF) {
    return a * DF - a * (a - 1) / 2 + (b - a);
}

template <int DF>
__device__ __forceinline__ float phi_sym(const float* x, int f, const unsigned char* pa,
                                         const unsigned char* pb) {
    if (f == 0) return 1.0f;
    if (f <= DF) return x[f - 1];
    const int a = pa[f], b = pb[f];
    const float p = x[a] * x[b];
    return a == b ? p * kSqrtHalf : p;
}

template <int DF, int C>
struct SimtSmem {
    static constexpr int DS = sym_feature_dim(DF);
    static constexpr int kQ = 0;
    static constexpr int kK = kQ + C * DF;
    static constexpr int kV = kK + C * DF;
    static constexpr int kA = kV + C * kCW;
    static constexpr int kPq = kA + C * (C + 1);
    static constexpr int kPk = kPq + C * DS;
    static constexpr int kS = kPk + C * DS;
    static constexpr int kZ = kS + DS * kCW;
    static constexpr int kDen = kZ + DS;
    static constexpr int kFloats = kDen + C;
    static constexpr size_t bytes = kFloats * sizeof(float) + 2 * DS;   // + pair tables
};

template <typename T, int DF, int DV, int C>
__global__ void __launch_bounds__(kThreads)
la_prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                       T* __restrict__ y, float* __restrict__ S, float* __restrict__ z, int N, int packed,
                       const float* __restrict__ gamma) {
    using L = SimtSmem<DF, C>;
    constexpr int DS = L::DS;
    constexpr int D = feature_dim(DF);
    extern __shared__ float smem[];
    float* sQ = smem + L::kQ;
    float* sK = smem + L::kK;
    float* sV = smem + L::kV;
    float* sA = smem + L::kA;
    float* sPq = smem + L::kPq;
    float* sPk = smem + L::kPk;
    float* sS = smem + L::kS;
    float* sz = smem + L::kZ;
    float* sden = smem + L::kDen;
    unsigned char* pa = reinterpret_cast<unsigned char*>(smem + L::kFloats);
    unsigned char* pb = pa + DS;

    const int tid = threadIdx.x;
    const size_t bh = blockIdx.y;
    const int c0 = blockIdx.x * kCW;

    if (tid == 0) {
        int f = 1 + DF;
        for (int a = 0; a < DF; ++a)
            for (int b = a; b < DF; ++b, ++f) { pa[f] = (unsigned char)a; pb[f] = (unsigned char)b; }
    }
    for (int e = tid; e < DS * kCW; e += kThreads) sS[e] = 0.f;
    for (int e = tid; e < DS; e += kThreads) sz[e] = 0.f;
    __syncthreads();

    const T* qb = q + bh * (size_t)N * DF;
    const T* kb = k + bh * (size_t)N * DF;
    const T* vb = v + bh * (size_t)N * DV;
    T* yb = y + bh * (size_t)N * DV;

    // Coarse decay: gamma of each 128-token tile scales the state where the tile
    // begins (a chunk of C <= 128 tokens never spans two tiles).
    const float* gh = gamma != nullptr ? gamma + bh * (size_t)((N + 127) / 128) : nullptr;
    for (int t0 = 0; t0 < N; t0 += C) {
        const int nv = min(C, N - t0);
        if (gh != nullptr && t0 > 0 && t0 % 128 == 0) {
            const float g = gh[t0 / 128];
            for (int e = tid; e < DS * kCW; e += kThreads) sS[e] *= g;
            for (int e = tid; e < DS; e += kThreads) sz[e] *= g;
        }
        for (int e = tid; e < C * DF; e += kThreads) {
            const int t = e / DF;
            const bool ok = t < nv;
            sQ[e] = ok ? to_f32(qb[(size_t)t0 * DF + e]) : 0.f;
            sK[e] = ok ? to_f32(kb[(size_t)t0 * DF + e]) : 0.f;
        }
        for (int e = tid; e < C * kCW; e += kThreads) {
            const int t = e / kCW, cc = e % kCW;
            sV[e] = t < nv ? to_f32(vb[(size_t)(t0 + t) * DV + c0 + cc]) : 0.f;
        }
        __syncthreads();
        for (int e = tid; e < C * DS; e += kThreads) {
            const int t = e / DS, f = e % DS;
            sPq[e] = phi_sym<DF>(sQ + t * DF, f, pa, pb);
            sPk[e] = t < nv ? phi_sym<DF>(sK + t * DF, f, pa, pb) : 0.f;   // padded tokens add nothing
        }
        for (int e = tid; e < C * C; e += kThreads) {
            const int i = e / C, j = e % C;
            float a = 0.f;
            if (j <= i) {
                float s = 0.f;
#pragma unroll
                for (int d = 0; d < DF; ++d) s = fmaf(sQ[i * DF + d], sK[j * DF + d], s);
                a = 1.f + s + 0.5f * s * s;
            }
            sA[i * (C + 1) + j] = a;
        }
        __syncthreads();
        if (tid < C) {
            float d = 0.f;
            for (int j = 0; j <= tid; ++j) d += sA[tid * (C + 1) + j];
            for (int f = 0; f < DS; ++f) d = fmaf(sPq[tid * DS + f], sz[f], d);
            sden[tid] = d;
        }
        __syncthreads();
        for (int e = tid; e < C * kCW; e += kThreads) {
            const int i = e / kCW, cc = e % kCW;
            if (i < nv) {
                float n = 0.f;
                for (int j = 0; j <= i; ++j) n = fmaf(sA[i * (C + 1) + j], sV[j * kCW + cc], n);
                for (int f = 0; f < DS; ++f) n = fmaf(sPq[i * DS + f], sS[f * kCW + cc], n);
                yb[(size_t)(t0 + i) * DV + c0 + cc] = from_f32<T>(n / sden[i]);
            }
        }
        __syncthreads();
        for (int e = tid; e < DS * kCW; e += kThreads) {
            const int f = e / kCW, cc = e % kCW;
            float acc = sS[e];
            for (int t = 0; t < C; ++t) acc = fmaf(sPk[t * DS + f], sV[t * kCW + cc], acc);
            sS[e] = acc;
        }
        for (int f = tid; f < DS; f += kThreads) {
            float acc = sz[f];
            for (int t = 0; t < C; ++t) acc += sPk[t * DS + f];
            sz[f] = acc;
        }
        __syncthreads();
    }

    if (S != nullptr && packed) {
        // The symmetric layout is the kernel's own: row f of S and z as accumulated.
        float* Sb = S + bh * (size_t)DS * DV;
        for (int e = tid; e < DS * kCW; e += kThreads) {
            const int ff = e / kCW, cc = e % kCW;
            Sb[(size_t)ff * DV + c0 + cc] = sS[ff * kCW + cc];
        }
        if (blockIdx.x == 0) {
            float* zb = z + bh * (size_t)DS;
            for (int ff = tid; ff < DS; ff += kThreads) zb[ff] = sz[ff];
        }
    } else if (S != nullptr) {
        float* Sb = S + bh * (size_t)D * DV;
        for (int e = tid; e < D * kCW; e += kThreads) {
            const int ff = e / kCW, cc = e % kCW;
            float val;
            if (ff <= DF) {
                val = sS[ff * kCW + cc];
            } else {
                const int p = ff - 1 - DF, a = p / DF, b = p % DF;
                const int lo = min(a, b), hi = max(a, b);
                const float s = sS[(1 + DF + pair_index(lo, hi, DF)) * kCW + cc];
                val = (a == b) ? s : s * kSqrtHalf;
            }
            Sb[(size_t)ff * DV + c0 + cc] = val;
        }
        if (blockIdx.x == 0) {
            float* zb = z + bh * (size_t)D;
            for (int ff = tid; ff < D; ff += kThreads) {
                float val;
                if (ff <= DF) {
                    val = sz[ff];
                } else {
                    const int p = ff - 1 - DF, a = p / DF, b = p % DF;
                    const int lo = min(a, b), hi = max(a, b);
                    const float s = sz[1 + DF + pair_index(lo, hi, DF)];
                    val = (a == b) ? s : s * kSqrtHalf;
                }
                zb[ff] = val;
            }
        }
    }
}

template <typename T, int DF, int DV, int C>
cudaError_t launch_c(const LaPrefillArgs& a, cudaStream_t stream) {
    constexpr size_t smem = SimtSmem<DF, C>::bytes;
    static_assert(smem <= 227 * 1024, "shared memory");
    auto kern = la_prefill_simt_kernel<T, DF, DV, C>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid(DV / kCW, a.B * a.H);
    kern<<<grid, kThreads, smem, stream>>>(static_cast<const T*>(a.q), static_cast<const T*>(a.k),
                                          static_cast<const T*>(a.v), static_cast<T*>(a.y), a.S, a.z,
                                          a.N, a.packed ? 1 : 0, a.gamma);
    return cudaGetLastError();
}

template <typename T, int DF, int DV>
cudaError_t launch_dims(const LaPrefillArgs& a, cudaStream_t stream) {
    switch (a.chunk) {
        case 16: return launch_c<T, DF, DV, 16>(a, stream);
        case 32: return launch_c<T, DF, DV, 32>(a, stream);
        case 64:
            if constexpr (DF <= 16) return launch_c<T, DF, DV, 64>(a, stream);
            return cudaErrorInvalidValue;
        default: return cudaErrorInvalidValue;
    }
}

template <typename T>
cudaError_t launch_t(const LaPrefillArgs& a, cudaStream_t stream) {
    if (a.d_feat == 16 && a.d_v == 64) return launch_dims<T, 16, 64>(a, stream);
    if (a.d_feat == 16 && a.d_v == 128) return launch_dims<T, 16, 128>(a, stream);
    if (a.d_feat == 32 && a.d_v == 64) return launch_dims<T, 32, 64>(a, stream);
    if (a.d_feat == 32 && a.d_v == 128) return launch_dims<T, 32, 128>(a, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_la_prefill_simt(const LaPrefillArgs& a, cudaStream_t stream) {
    return a.bf16 ? launch_t<__nv_bfloat16>(a, stream) : launch_t<float>(a, stream);
}

}  // namespace based

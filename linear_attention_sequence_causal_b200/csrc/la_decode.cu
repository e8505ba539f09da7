// Recurrent (next-token) step of causal Taylor linear attention.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), §2 "Efficient attentions" (recurrent generation at O(1)
// per token) and App. B "Next Token Prediction" (KV-state update kernel):
//     S += phi(k) v^T,  z += phi(k),  y = phi(q)^T S / phi(q)^T z.
//
// The step is bound by HBM: each (b, h) reads and writes its fp32 state once
// (D x dv + D floats, 70 KB at d' = 16, dv = 64) while doing ~0.5 flop per byte.
// One CTA streams one head's S with 128-bit loads and stores; consecutive
// threads cover consecutive 16-byte pieces of a row, so a warp touches whole
// row segments. phi(q) and phi(k) are formed once per CTA in shared memory and
// never reach HBM. A head is never split across CTAs: z is updated in place and
// every CTA that read it would race with the one writing it. Small batches get
// larger CTAs (up to 1024 threads) instead, to keep enough loads in flight.
#include "common.cuh"
#include "kernels.h"

namespace based {
namespace {

template <int DF>
__device__ __forceinline__ float phi_entry(const float* x, int f) {
    if (f == 0) return 1.0f;
    if (f <= DF) return x[f - 1];
    const int p = f - 1 - DF;
    return (x[p / DF] * x[p % DF]) * kSqrtHalf;
}

template <typename T, int DF, int DV, int NT>
__global__ void __launch_bounds__(NT)
la_decode_kernel(float* __restrict__ S, float* __restrict__ z, const T* __restrict__ q,
                 const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ y) {
    constexpr int D = feature_dim(DF);
    constexpr int CW = DV;
    constexpr int G = CW / 4;          // float4 pieces per row
    constexpr int R = NT / G;          // rows in flight per sweep
    constexpr int kThreads = NT;
    static_assert(NT % G == 0 && NT >= CW, "thread layout");

    __shared__ float s_x[2][DF];
    __shared__ float s_fq[D];
    __shared__ float s_fk[D];
    __shared__ float s_v[CW];
    __shared__ float4 s_red[R][G];
    __shared__ float s_dred[kThreads / 32];

    const int tid = threadIdx.x;
    const size_t bh = blockIdx.x;

    if (tid < DF) {
        s_x[0][tid] = to_f32(q[bh * DF + tid]);
        s_x[1][tid] = to_f32(k[bh * DF + tid]);
    }
    if (tid < CW) s_v[tid] = to_f32(v[bh * DV + tid]);
    __syncthreads();
    for (int f = tid; f < D; f += kThreads) {
        s_fq[f] = phi_entry<DF>(s_x[0], f);
        s_fk[f] = phi_entry<DF>(s_x[1], f);
    }
    __syncthreads();

    // Denominator phi(q).z_new over all D features; z_new written back in place.
    float dpart = 0.f;
    float* zbh = z + bh * D;
    for (int f = tid; f < D; f += kThreads) {
        const float zn = zbh[f] + s_fk[f];
        zbh[f] = zn;
        dpart = fmaf(s_fq[f], zn, dpart);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dpart += __shfl_xor_sync(0xffffffffu, dpart, o);
    if ((tid & 31) == 0) s_dred[tid >> 5] = dpart;

    // Stream the state: one read, one write per element.
    const int g = tid % G;
    const int r0 = tid / G;
    const float4 vv = make_float4(s_v[4 * g], s_v[4 * g + 1], s_v[4 * g + 2], s_v[4 * g + 3]);
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float* Sp = S + bh * (size_t)D * DV + 4 * g;
#pragma unroll 4
    for (int f = r0; f < D; f += R) {
        float4* p = reinterpret_cast<float4*>(Sp + (size_t)f * DV);
        float4 s = __ldcs(p);
        const float kf = s_fk[f];
        const float qf = s_fq[f];
        s.x = fmaf(kf, vv.x, s.x);
        s.y = fmaf(kf, vv.y, s.y);
        s.z = fmaf(kf, vv.z, s.z);
        s.w = fmaf(kf, vv.w, s.w);
        __stcs(p, s);
        acc.x = fmaf(qf, s.x, acc.x);
        acc.y = fmaf(qf, s.y, acc.y);
        acc.z = fmaf(qf, s.z, acc.z);
        acc.w = fmaf(qf, s.w, acc.w);
    }
    s_red[r0][g] = acc;
    __syncthreads();
    if (tid < CW) {
        float den = 0.f;
#pragma unroll
        for (int i = 0; i < kThreads / 32; ++i) den += s_dred[i];
        const int gg = tid >> 2, comp = tid & 3;
        float num = 0.f;
#pragma unroll 8
        for (int r = 0; r < R; ++r) num += reinterpret_cast<const float*>(&s_red[r][gg])[comp];
        y[bh * DV + tid] = from_f32<T>(num / den);
    }
}

template <typename T, int DF, int DV>
cudaError_t launch_typed(float* S, float* z, const void* q, const void* k, const void* v, void* y,
                         int BH, int num_sms, cudaStream_t stream) {
    auto qq = static_cast<const T*>(q);
    auto kk = static_cast<const T*>(k);
    auto vv = static_cast<const T*>(v);
    auto yy = static_cast<T*>(y);
    // One CTA per head; fewer heads than ~2 waves of SMs get wider CTAs.
    if ((long long)BH >= 2LL * num_sms)
        la_decode_kernel<T, DF, DV, 256><<<BH, 256, 0, stream>>>(S, z, qq, kk, vv, yy);
    else if ((long long)BH >= num_sms / 2)
        la_decode_kernel<T, DF, DV, 512><<<BH, 512, 0, stream>>>(S, z, qq, kk, vv, yy);
    else
        la_decode_kernel<T, DF, DV, 1024><<<BH, 1024, 0, stream>>>(S, z, qq, kk, vv, yy);
    return cudaGetLastError();
}

template <typename T>
cudaError_t dispatch(float* S, float* z, const void* q, const void* k, const void* v, void* y,
                     int BH, int d_feat, int d_v, int num_sms, cudaStream_t stream) {
    if (d_feat == 16 && d_v == 64) return launch_typed<T, 16, 64>(S, z, q, k, v, y, BH, num_sms, stream);
    if (d_feat == 16 && d_v == 128) return launch_typed<T, 16, 128>(S, z, q, k, v, y, BH, num_sms, stream);
    if (d_feat == 32 && d_v == 64) return launch_typed<T, 32, 64>(S, z, q, k, v, y, BH, num_sms, stream);
    if (d_feat == 32 && d_v == 128) return launch_typed<T, 32, 128>(S, z, q, k, v, y, BH, num_sms, stream);
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_la_decode(float* S, float* z, const void* q, const void* k, const void* v,
                             void* y, int B, int H, int d_feat, int d_v, bool bf16, int num_sms,
                             cudaStream_t stream) {
    const int BH = B * H;
    return bf16 ? dispatch<__nv_bfloat16>(S, z, q, k, v, y, BH, d_feat, d_v, num_sms, stream)
                : dispatch<float>(S, z, q, k, v, y, BH, d_feat, d_v, num_sms, stream);
}

}  // namespace based

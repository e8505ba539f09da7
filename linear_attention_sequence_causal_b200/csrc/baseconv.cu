// Short gated convolution (BaseConv) mixing core: causal depthwise K-tap filter,
// SiLU on the filtered branch, Hadamard gate.
//
// BASED ("Simple linear attention language models balance the recall-throughput
// tradeoff") §4 "The BASED Architecture" (Additional mixers) and App. C
// "Extended Architecture Details" (Convolution): a short convolution and a SiLU
// combined with the projected input by an elementwise product. For the two
// projected streams u_gate, u_conv [B, N, d] (channels innermost):
//     c_t = bias + sum_{j<K} h[:, j] * u_conv[t - (K-1) + j]   (zero before token 0)
//     y_t = u_gate[t] * SiLU(c_t)
// The work is a few FMAs per element against 3 element transfers, so both
// kernels are bound by HBM: the design goal is to move each element once, in
// 16-byte coalesced pieces, with enough loads in flight to cover DRAM latency.
//
// Prefill: one thread owns V consecutive channels (8 of bf16 when d allows,
// else 4) of one sequence over a run of `seg` tokens, `seg` chosen so that the
// grid fills the resident thread slots once. It keeps the last K-1 values of
// u_conv in registers (a sliding window), so every u_conv element is read once
// plus a K-1 token halo per run (served by L2: the neighbouring run read it
// from DRAM). Consecutive threads own consecutive channel groups, so a warp
// reads 512 contiguous bytes of a token row per stream (256 with 4 bf16
// channels). The streams reach shared memory by cp.async in stages of 4
// tokens, 2 or 3 stages in flight while the thread computes one, so DRAM
// latency is covered without holding the data in registers. The run that ends
// the sequence writes the generation state (the last K-1 values of u_conv,
// oldest first).
//
// Decode: one thread per (sequence, 4 channels): read the K-1 state rows and
// the new token, write y and the shifted state in place. No thread reads what
// another writes.
#include <cuda_bf16.h>
#include <stdint.h>

#include <algorithm>
#include <atomic>

#include "common.cuh"
#include "kernels.h"

namespace based {
namespace {

constexpr int kUnroll = 4;           // tokens per ring stage
constexpr int kThreads = 128;        // prefill block
constexpr int kDecodeThreads = 64;   // decode block: small batches still spread over many SMs

// V channels of one token of the dtype: 8 bytes (bf16, V = 4) or 16 bytes
// (bf16, V = 8; fp32, V = 4), moved as one vector.
template <bool BF16, int V> struct Piece;
template <> struct Piece<true, 4> { using raw = uint2; };
template <> struct Piece<true, 8> { using raw = uint4; };
template <> struct Piece<false, 4> { using raw = uint4; };
template <bool BF16, int V> using Raw = typename Piece<BF16, V>::raw;

template <bool BF16, int V>
__device__ __forceinline__ const Raw<BF16, V>* at(const void* base, size_t off) {
    if constexpr (BF16) return reinterpret_cast<const Raw<BF16, V>*>(static_cast<const __nv_bfloat16*>(base) + off);
    else return reinterpret_cast<const Raw<BF16, V>*>(static_cast<const float*>(base) + off);
}

template <bool BF16, int V>
__device__ __forceinline__ Raw<BF16, V>* at(void* base, size_t off) {
    if constexpr (BF16) return reinterpret_cast<Raw<BF16, V>*>(static_cast<__nv_bfloat16*>(base) + off);
    else return reinterpret_cast<Raw<BF16, V>*>(static_cast<float*>(base) + off);
}

template <bool BF16, int V>
__device__ __forceinline__ void to_float(const Raw<BF16, V>& r, float (&x)[V]) {
    if constexpr (BF16) {
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&r);
#pragma unroll
        for (int i = 0; i < V / 2; ++i) {
            const float2 f = __bfloat1622float2(p[i]);
            x[2 * i] = f.x;
            x[2 * i + 1] = f.y;
        }
    } else {
        const float* p = reinterpret_cast<const float*>(&r);
#pragma unroll
        for (int i = 0; i < V; ++i) x[i] = p[i];
    }
}

template <bool BF16, int V>
__device__ __forceinline__ Raw<BF16, V> from_float(const float (&x)[V]) {
    Raw<BF16, V> r;
    if constexpr (BF16) {
        __nv_bfloat162* p = reinterpret_cast<__nv_bfloat162*>(&r);
#pragma unroll
        for (int i = 0; i < V / 2; ++i) p[i] = __floats2bfloat162_rn(x[2 * i], x[2 * i + 1]);
    } else {
        float* p = reinterpret_cast<float*>(&r);
#pragma unroll
        for (int i = 0; i < V; ++i) p[i] = x[i];
    }
    return r;
}

// Read-only inputs: through the non-coherent path.
template <bool BF16, int V>
__device__ __forceinline__ void load_ro(const void* base, size_t off, float (&x)[V]) {
    to_float<BF16, V>(__ldg(at<BF16, V>(base, off)), x);
}

// Plain load, for the decode state that the same kernel rewrites.
template <bool BF16, int V>
__device__ __forceinline__ void load_rw(const void* base, size_t off, float (&x)[V]) {
    to_float<BF16, V>(*at<BF16, V>(base, off), x);
}

template <bool BF16, int V>
__device__ __forceinline__ void store(void* base, size_t off, const float (&x)[V]) {
    *at<BF16, V>(base, off) = from_float<BF16, V>(x);
}

template <bool BF16, int V>
__device__ __forceinline__ void copy_async(Raw<BF16, V>* dst, const void* base, size_t off) {
    const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(dst));
    const void* src = at<BF16, V>(base, off);
    if constexpr (sizeof(Raw<BF16, V>) == 16)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(src) : "memory");
    else
        asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s), "l"(src) : "memory");
}

// Ring depth: 4 stages of 8-byte pieces (32 KB per block), 3 of 16-byte pieces (48 KB).
template <bool BF16, int V> constexpr int kStages = sizeof(Raw<BF16, V>) == 16 ? 3 : 4;

// x * sigmoid(x). For x < -87, exp(-x) exceeds 2^126 and the fast divide returns 0,
// the limit of the function there.
__device__ __forceinline__ float silu(float c) { return __fdividef(c, 1.0f + __expf(-c)); }

// The K taps of V consecutive channels are VK consecutive floats of h [d, K],
// 16-byte aligned because the first channel is a multiple of V (4 or 8).
template <int K, int V>
__device__ __forceinline__ void load_filter(const float* __restrict__ h, const float* __restrict__ bias,
                                            int c0, float (&hr)[K][V], float (&br)[V]) {
    const float4* hp = reinterpret_cast<const float4*>(h + (size_t)c0 * K);
    float flat[V * K];
#pragma unroll
    for (int i = 0; i < V * K / 4; ++i) {
        const float4 f = __ldg(hp + i);
        flat[4 * i] = f.x; flat[4 * i + 1] = f.y; flat[4 * i + 2] = f.z; flat[4 * i + 3] = f.w;
    }
#pragma unroll
    for (int e = 0; e < V; ++e)
#pragma unroll
        for (int j = 0; j < K; ++j) hr[j][e] = flat[e * K + j];
    if (bias != nullptr) {
#pragma unroll
        for (int i = 0; i < V / 4; ++i) {
            const float4 b = __ldg(reinterpret_cast<const float4*>(bias + c0) + i);
            br[4 * i] = b.x; br[4 * i + 1] = b.y; br[4 * i + 2] = b.z; br[4 * i + 3] = b.w;
        }
    } else {
#pragma unroll
        for (int e = 0; e < V; ++e) br[e] = 0.0f;
    }
}

// Resident blocks per SM asked of the compiler: the most that keeps the filter
// and the window in registers without spilling and that the ring's shared
// memory allows (6 blocks of 4-channel threads at K = 3 or 4; 4 blocks of
// 8-channel threads, whose 48 KB rings allow no more).
constexpr int prefill_min_blocks(int K, bool bf16, int V) {
    return V == 8 ? 4 : K <= 2 ? 8 : K <= 3 ? 6 : K == 4 ? (bf16 ? 6 : 5) : K <= 6 ? 4 : 3;
}

template <int K, bool BF16, int V>
__global__ void __launch_bounds__(kThreads, prefill_min_blocks(K, BF16, V))
baseconv_prefill_kernel(const void* __restrict__ gate, const void* __restrict__ conv,
                        const float* __restrict__ h, const float* __restrict__ bias, void* __restrict__ y,
                        void* __restrict__ state, int N, int d, int seg, int nseg, int groups, int items,
                        unsigned* status, size_t y_elems, size_t state_elems) {
    constexpr int S = kStages<BF16, V>;
    const int item = blockIdx.x * kThreads + threadIdx.x;
    if (item >= items) return;
    const int cg = item % groups;
    const int rest = item / groups;
    const int s = rest % nseg;
    const int b = rest / nseg;
    const int c0 = cg * V;
    const int t0 = s * seg;
    const int t1 = min(N, t0 + seg);
    const size_t row0 = (size_t)b * N;

    // Async-copy ring: stage q holds tokens t0 + q*kUnroll .. +kUnroll-1 of both
    // streams in slot q % S. Each thread copies and later reads only its own
    // entries (column threadIdx.x), so the only wait is cp.async.wait_group on
    // its own copies; S-1 stages stay in flight while one is computed.
    __shared__ Raw<BF16, V> ring[S][kUnroll][2][kThreads];
    const int tid = threadIdx.x;
    const int nstage = (t1 - t0 + kUnroll - 1) / kUnroll;
    auto issue = [&](int q) {
        if (q < nstage) {
            const int slot = q % S;
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int t = t0 + q * kUnroll + u;
                if (t < t1) {
                    const size_t off = (row0 + t) * d + c0;
                    copy_async<BF16, V>(&ring[slot][u][0][tid], gate, off);
                    copy_async<BF16, V>(&ring[slot][u][1][tid], conv, off);
                }
            }
        }
        asm volatile("cp.async.commit_group;\n" ::: "memory");
    };
#pragma unroll
    for (int q = 0; q < S - 1; ++q) issue(q);

    float hr[K][V], br[V];
    load_filter<K, V>(h, bias, c0, hr, br);

    // win[j] holds u_conv of token t - (K-1) + j for the token t about to be processed.
    float win[K > 1 ? K - 1 : 1][V];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) {
        const int t = t0 - (K - 1) + j;
        if (t >= 0) {
            load_ro<BF16, V>(conv, (row0 + t) * d + c0, win[j]);
        } else {
#pragma unroll
            for (int e = 0; e < V; ++e) win[j][e] = 0.0f;
        }
    }

    for (int q = 0; q < nstage; ++q) {
        issue(q + S - 1);
        asm volatile("cp.async.wait_group %0;\n" ::"n"(S - 1) : "memory");
        const int slot = q % S;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int t = t0 + q * kUnroll + u;
            if (t < t1) {
                float g[V], x[V], out[V];
                to_float<BF16, V>(ring[slot][u][0][tid], g);
                to_float<BF16, V>(ring[slot][u][1][tid], x);
#pragma unroll
                for (int e = 0; e < V; ++e) {
                    float c = br[e];
#pragma unroll
                    for (int j = 0; j < K - 1; ++j) c = fmaf(hr[j][e], win[j][e], c);
                    c = fmaf(hr[K - 1][e], x[e], c);
                    out[e] = g[e] * silu(c);
                }
                if (in_bounds((row0 + t) * d + c0 + V - 1, y_elems, status)) store<BF16, V>(y, (row0 + t) * d + c0, out);
#pragma unroll
                for (int j = 0; j + 1 < K - 1; ++j)
#pragma unroll
                    for (int e = 0; e < V; ++e) win[j][e] = win[j + 1][e];
                if constexpr (K > 1) {
#pragma unroll
                    for (int e = 0; e < V; ++e) win[K - 2][e] = x[e];
                }
            }
        }
    }

    // The window now holds tokens N-K+1 .. N-1 (zeros before token 0).
    if (state != nullptr && t1 == N) {
#pragma unroll
        for (int j = 0; j < K - 1; ++j)
            if (in_bounds(((size_t)b * (K - 1) + j) * d + c0 + V - 1, state_elems, status))
                store<BF16, V>(state, ((size_t)b * (K - 1) + j) * d + c0, win[j]);
    }
}

constexpr int kDecodeVec = 4;   // channels per decode thread

template <int K, bool BF16>
__global__ void __launch_bounds__(kDecodeThreads)
baseconv_decode_kernel(void* __restrict__ state, const void* __restrict__ gate, const void* __restrict__ conv,
                       const float* __restrict__ h, const float* __restrict__ bias, void* __restrict__ y,
                       int d, int groups, int items, unsigned* status, size_t y_elems, size_t state_elems) {
    constexpr int V = kDecodeVec;
    const int item = blockIdx.x * kDecodeThreads + threadIdx.x;
    if (item >= items) return;
    const int cg = item % groups;
    const int b = item / groups;
    const int c0 = cg * V;

    float hr[K][V], br[V];
    load_filter<K, V>(h, bias, c0, hr, br);

    float st[K > 1 ? K - 1 : 1][V];
#pragma unroll
    for (int j = 0; j < K - 1; ++j) load_rw<BF16, V>(state, ((size_t)b * (K - 1) + j) * d + c0, st[j]);
    float g[V], x[V];
    load_ro<BF16, V>(gate, (size_t)b * d + c0, g);
    load_ro<BF16, V>(conv, (size_t)b * d + c0, x);

    float out[V];
#pragma unroll
    for (int e = 0; e < V; ++e) {
        float c = br[e];
#pragma unroll
        for (int j = 0; j < K - 1; ++j) c = fmaf(hr[j][e], st[j][e], c);
        c = fmaf(hr[K - 1][e], x[e], c);
        out[e] = g[e] * silu(c);
    }
    if (in_bounds((size_t)b * d + c0 + V - 1, y_elems, status)) store<BF16, V>(y, (size_t)b * d + c0, out);
    if constexpr (K > 1) {
        if (!in_bounds(((size_t)b * (K - 1) + (K - 2)) * d + c0 + V - 1, state_elems, status)) return;
#pragma unroll
        for (int j = 0; j + 1 < K - 1; ++j) store<BF16, V>(state, ((size_t)b * (K - 1) + j) * d + c0, st[j + 1]);
        store<BF16, V>(state, ((size_t)b * (K - 1) + (K - 2)) * d + c0, x);
    }
}

// Token run per thread: split each (sequence, channel group) column into as
// many runs as the resident thread slots allow, so that the grid is one wave
// of equal runs (no tail) with the fewest halo re-reads.
int prefill_segment(int B, int N, int groups, long long slots) {
    const long long columns = (long long)B * groups;
    const long long runs = std::max(1LL, std::min<long long>(N, slots / columns));
    return (int)((N + runs - 1) / runs);
}

template <int K, bool BF16, int V>
cudaError_t prefill_k(cudaStream_t st, const void* gate, const void* conv, const float* h, const float* bias,
                      void* y, void* state, int B, int N, int d, int num_sms, unsigned* status) {
    // Resident blocks per SM, a property of the compiled kernel on a device:
    // looked up once per device (the carveout attribute is set per device too).
    constexpr int kDevices = 64;
    static std::atomic<int> occ[kDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kDevices) return cudaErrorInvalidDevice;
    int occupancy = occ[dev].load(std::memory_order_relaxed);
    if (occupancy == 0) {
        // the ring lives in shared memory: prefer the largest shared-memory carveout
        cudaError_t e = cudaFuncSetAttribute(baseconv_prefill_kernel<K, BF16, V>,
                                             cudaFuncAttributePreferredSharedMemoryCarveout,
                                             cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
        int o = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&o, baseconv_prefill_kernel<K, BF16, V>, kThreads, 0);
        if (e != cudaSuccess) return e;
        occupancy = std::max(1, o);
        occ[dev].store(occupancy, std::memory_order_relaxed);   // same value from every racing thread
    }
    const int groups = d / V;
    const int seg = prefill_segment(B, N, groups, (long long)num_sms * occupancy * kThreads);
    const int nseg = (N + seg - 1) / seg;
    const long long items = (long long)B * nseg * groups;
    if (items > 0x7fffffffLL - kThreads) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)((items + kThreads - 1) / kThreads));
    baseconv_prefill_kernel<K, BF16, V><<<grid, kThreads, 0, st>>>(gate, conv, h, bias, y, state, N, d, seg,
                                                                    nseg, groups, (int)items, status,
                                                                    (size_t)B * N * d, (size_t)B * (K - 1) * d);
    return cudaGetLastError();
}

template <int K, bool BF16>
cudaError_t decode_k(cudaStream_t st, void* state, const void* gate, const void* conv, const float* h,
                     const float* bias, void* y, int B, int d, unsigned* status) {
    const int groups = d / kDecodeVec;
    const long long items = (long long)B * groups;
    if (items > 0x7fffffffLL - kDecodeThreads) return cudaErrorInvalidValue;
    const dim3 grid((unsigned)((items + kDecodeThreads - 1) / kDecodeThreads));
    baseconv_decode_kernel<K, BF16><<<grid, kDecodeThreads, 0, st>>>(state, gate, conv, h, bias, y, d, groups,
                                                                      (int)items, status, (size_t)B * d,
                                                                      (size_t)B * (K - 1) * d);
    return cudaGetLastError();
}

// 16-byte pieces (8 bf16 channels) when the channel count allows and the filter
// is short enough for 8 channels of taps and window to stay in registers, else
// 4 channels.
template <int K, bool BF16>
cudaError_t prefill_v(cudaStream_t st, const void* gate, const void* conv, const float* h, const float* bias,
                      void* y, void* state, int B, int N, int d, int num_sms, unsigned* status) {
    if constexpr (BF16 && K <= 5) {
        if (d % 8 == 0) return prefill_k<K, true, 8>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
    }
    return prefill_k<K, BF16, 4>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
}

template <bool BF16>
cudaError_t prefill_any(int K, cudaStream_t st, const void* gate, const void* conv, const float* h,
                        const float* bias, void* y, void* state, int B, int N, int d, int num_sms,
                        unsigned* status) {
    switch (K) {
        case 1: return prefill_v<1, BF16>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
        case 2: return prefill_v<2, BF16>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
        case 3: return prefill_v<3, BF16>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
        case 4: return prefill_v<4, BF16>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
        case 5: return prefill_v<5, BF16>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
        case 6: return prefill_v<6, BF16>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
        case 7: return prefill_v<7, BF16>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
        case 8: return prefill_v<8, BF16>(st, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
        default: return cudaErrorInvalidValue;
    }
}

template <bool BF16>
cudaError_t decode_any(int K, cudaStream_t st, void* state, const void* gate, const void* conv, const float* h,
                       const float* bias, void* y, int B, int d, unsigned* status) {
    switch (K) {
        case 1: return decode_k<1, BF16>(st, state, gate, conv, h, bias, y, B, d, status);
        case 2: return decode_k<2, BF16>(st, state, gate, conv, h, bias, y, B, d, status);
        case 3: return decode_k<3, BF16>(st, state, gate, conv, h, bias, y, B, d, status);
        case 4: return decode_k<4, BF16>(st, state, gate, conv, h, bias, y, B, d, status);
        case 5: return decode_k<5, BF16>(st, state, gate, conv, h, bias, y, B, d, status);
        case 6: return decode_k<6, BF16>(st, state, gate, conv, h, bias, y, B, d, status);
        case 7: return decode_k<7, BF16>(st, state, gate, conv, h, bias, y, B, d, status);
        case 8: return decode_k<8, BF16>(st, state, gate, conv, h, bias, y, B, d, status);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_baseconv_prefill(const void* gate, const void* conv, const float* h, const float* bias,
                                    void* y, void* state, int B, int N, int d, int K, bool bf16, int num_sms,
                                    unsigned* status, cudaStream_t stream) {
    if (B <= 0 || N <= 0 || d <= 0 || d % 4 != 0 || K < 1 || K > kMaxConvTaps || num_sms <= 0)
        return cudaErrorInvalidValue;
    return bf16 ? prefill_any<true>(K, stream, gate, conv, h, bias, y, state, B, N, d, num_sms, status)
                : prefill_any<false>(K, stream, gate, conv, h, bias, y, state, B, N, d, num_sms, status);
}

cudaError_t launch_baseconv_decode(void* state, const void* gate, const void* conv, const float* h,
                                   const float* bias, void* y, int B, int d, int K, bool bf16,
                                   unsigned* status, cudaStream_t stream) {
    if (B <= 0 || d <= 0 || d % kDecodeVec != 0 || K < 1 || K > kMaxConvTaps) return cudaErrorInvalidValue;
    return bf16 ? decode_any<true>(K, stream, state, gate, conv, h, bias, y, B, d, status)
                : decode_any<false>(K, stream, state, gate, conv, h, bias, y, B, d, status);
}

}  // namespace based

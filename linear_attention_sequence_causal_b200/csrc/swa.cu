// Causal sliding-window softmax attention: prefill over a sequence, decode over a ring cache.
//
// "Simple linear attention language models balance the recall-throughput
// tradeoff" (BASED), §4 "Local Exact Attention": exact softmax over a window of
// the most recent keys, O(Nw) time and a w-sized KV cache for generation; App. B
// "Next Token Prediction" names the windowed decode as one of the generation
// kernels. Window convention: token i sees keys i - w < j <= i (w keys including
// itself), which is what a w-slot ring holds after token i is written.
//
// Prefill: bf16 inputs go to the tensor-core kernel (swa_tc.cu). The fp32
// path below runs on the CUDA cores: a CTA takes 64 consecutive queries of one head and
// stages those queries plus the 64 + w - 1 keys and values they can see in
// shared memory (fp32), so every K/V row is read from global memory once per
// tile. Four threads share a query, each owning 16 of the 64 dims: partial dot
// products are combined with two butterfly shuffles and the softmax runs online
// (running max and sum, rescaling the accumulator), in fp32 with expf.
//
// Decode: one CTA per (b, h); the new key/value go to slot t mod w. bf16 uses
// 16-byte loads (see the two swa_decode_bf16 kernels); the fp32 kernel scores slot j on
// thread j, reduces max and sum, then accumulates output dim e on thread e.
#include <math.h>

#include "common.cuh"
#include "kernels.h"
#include "tcgen05.cuh"

namespace based {
namespace {

constexpr int kQTile = 64;
constexpr int kHead = 64;        // head dim d
constexpr int kMaxW = 64;

// 16-byte asynchronous copy global -> shared (through L2, not L1), and the wait
// for all of this thread's copies.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Two floats as a bf16x2 word (round to nearest even), low half first.
__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

template <typename T>
__global__ void __launch_bounds__(256)
swa_prefill_simt_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                        T* __restrict__ y, int N, int w, float scale) {
    extern __shared__ float smem[];
    constexpr int KR = kQTile + kMaxW - 1;                 // key rows a tile can see
    float* sQ = smem;                                      // [64][64]
    float* sK = sQ + kQTile * kHead;                       // [KR][64]
    float* sV = sK + KR * kHead;                           // [KR][64]

    const int tid = threadIdx.x;
    const size_t bh = blockIdx.y;
    const int i0 = blockIdx.x * kQTile;
    const int j0 = i0 - (w - 1);                           // first key row (may be < 0)
    const T* qb = q + bh * (size_t)N * kHead;
    const T* kb = k + bh * (size_t)N * kHead;
    const T* vb = v + bh * (size_t)N * kHead;

    for (int e = tid; e < kQTile * kHead; e += 256) {
        const int r = e / kHead;
        sQ[e] = (i0 + r < N) ? to_f32(qb[(size_t)i0 * kHead + e]) : 0.f;
    }
    const int nk = kQTile + w - 1;
    for (int e = tid; e < nk * kHead; e += 256) {
        const int r = e / kHead, c = e % kHead;
        const int j = j0 + r;
        const bool ok = j >= 0 && j < N;
        sK[e] = ok ? to_f32(kb[(size_t)j * kHead + c]) : 0.f;
        sV[e] = ok ? to_f32(vb[(size_t)j * kHead + c]) : 0.f;
    }
    __syncthreads();

    const int qi = tid >> 2;          // query within the tile
    const int part = tid & 3;         // 16-dim slice
    const int i = i0 + qi;
    const float* qrow = sQ + qi * kHead + part * 16;
    float qreg[16];
#pragma unroll
    for (int d = 0; d < 16; ++d) qreg[d] = qrow[d] * scale;

    float m = -INFINITY, l = 0.f;
    float acc[16];
#pragma unroll
    for (int d = 0; d < 16; ++d) acc[d] = 0.f;

    // Same trip count for every lane (w), so the shuffles stay converged.
    for (int jj = 0; jj < w; ++jj) {
        const int j = i - jj;                              // key position
        const int r = j - j0;                              // row in sK / sV
        const bool valid = (j >= 0) && (i < N);
        const float* krow = sK + (valid ? r : 0) * kHead + part * 16;
        float s = 0.f;
#pragma unroll
        for (int d = 0; d < 16; ++d) s = fmaf(qreg[d], krow[d], s);
        s += __shfl_xor_sync(0xffffffffu, s, 1);
        s += __shfl_xor_sync(0xffffffffu, s, 2);
        if (valid) {
            const float mn = fmaxf(m, s);
            const float corr = expf(m - mn);               // 0 on the first key (m = -inf)
            const float p = expf(s - mn);
            l = l * corr + p;
            const float* vrow = sV + r * kHead + part * 16;
#pragma unroll
            for (int d = 0; d < 16; ++d) acc[d] = fmaf(p, vrow[d], acc[d] * corr);
            m = mn;
        }
    }
    if (i < N) {
        const float inv = 1.f / l;
        T* yrow = y + (bh * (size_t)N + i) * kHead + part * 16;
#pragma unroll
        for (int d = 0; d < 16; ++d) yrow[d] = from_f32<T>(acc[d] * inv);
    }
}

// Ring cache after the prompt: slot t mod w holds token t for t in [max(0, N-w), N), others 0.
template <typename T>
__global__ void swa_fill_ring_kernel(const T* __restrict__ k, const T* __restrict__ v,
                                     T* __restrict__ kc, T* __restrict__ vc, int N, int w) {
    const size_t bh = blockIdx.x;
    for (int e = threadIdx.x; e < w * kHead; e += blockDim.x) {
        const int slot = e / kHead, c = e % kHead;
        // newest token u < N with u mod w == slot
        const int last = N - 1;
        const int u = last - (((last - slot) % w) + w) % w;
        T kv = from_f32<T>(0.f), vv = from_f32<T>(0.f);
        if (u >= 0) {
            kv = k[(bh * (size_t)N + u) * kHead + c];
            vv = v[(bh * (size_t)N + u) * kHead + c];
        }
        kc[(bh * w + slot) * kHead + c] = kv;
        vc[(bh * w + slot) * kHead + c] = vv;
    }
}

template <typename T>
__global__ void __launch_bounds__(kMaxW)
swa_decode_kernel(T* __restrict__ kc, T* __restrict__ vc, long long t, const T* __restrict__ q,
                  const T* __restrict__ k, const T* __restrict__ v, T* __restrict__ y, int w,
                  float scale, unsigned* status) {
    __shared__ float s_q[kHead], s_k[kHead], s_v[kHead];
    __shared__ float s_p[kMaxW];
    __shared__ float s_red[2][2];
    const int tid = threadIdx.x;          // 64 threads
    const size_t bh = blockIdx.x;
    const int new_slot = (int)(t % w);

    s_q[tid] = to_f32(q[bh * kHead + tid]) * scale;
    const T knew = k[bh * kHead + tid];
    const T vnew = v[bh * kHead + tid];
    s_k[tid] = to_f32(knew);
    s_v[tid] = to_f32(vnew);
    __syncthreads();

    float s = -INFINITY;
    bool valid = false;
    if (tid < w) {
        // newest token u <= t held by slot tid; valid when u >= 0
        const long long u = t - ((((t - tid) % w) + w) % w);
        valid = u >= 0;
        if (valid) {
            float acc = 0.f;
            if (tid == new_slot) {
#pragma unroll 16
                for (int d = 0; d < kHead; ++d) acc = fmaf(s_q[d], s_k[d], acc);
            } else {
                const T* krow = kc + (bh * w + tid) * kHead;
#pragma unroll 16
                for (int d = 0; d < kHead; ++d) acc = fmaf(s_q[d], to_f32(krow[d]), acc);
            }
            s = acc;
        }
    }
    float m = s;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if ((tid & 31) == 0) s_red[0][tid >> 5] = m;
    __syncthreads();
    m = fmaxf(s_red[0][0], s_red[0][1]);
    const float p = valid ? expf(s - m) : 0.f;
    float sum = p;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    if ((tid & 31) == 0) s_red[1][tid >> 5] = sum;
    s_p[tid] = p;
    __syncthreads();
    const float inv = 1.f / (s_red[1][0] + s_red[1][1]);

    float acc = 0.f;
    for (int j = 0; j < w; ++j) {
        const float pj = s_p[j];
        if (pj != 0.f) {
            const float vj = (j == new_slot) ? s_v[tid] : to_f32(vc[(bh * w + j) * kHead + tid]);
            acc = fmaf(pj, vj, acc);
        }
    }
    const size_t n_heads = gridDim.x;                // extents of y and the ring for the index checks
    if (in_bounds(bh * kHead + tid, n_heads * kHead, status)) y[bh * kHead + tid] = from_f32<T>(acc * inv);
    const size_t slot_at = (bh * w + new_slot) * kHead + tid;
    if (in_bounds(slot_at, n_heads * w * kHead, status)) {
        kc[slot_at] = knew;
        vc[slot_at] = vnew;
    }
}

template <typename T>
cudaError_t prefill_t(const void* q, const void* k, const void* v, void* y, void* k_cache,
                      void* v_cache, int B, int H, int N, int w, float scale, unsigned* status,
                      unsigned debug, cudaStream_t stream) {
    if constexpr (sizeof(T) == 2) {
        return launch_swa_prefill_tc(q, k, v, y, k_cache, v_cache, B, H, N, w, scale, status, debug, stream);
    } else {
        constexpr size_t smem = (size_t)(kQTile * kHead + 2 * (kQTile + kMaxW - 1) * kHead) * sizeof(float);
        auto kern = swa_prefill_simt_kernel<T>;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        const dim3 grid((N + kQTile - 1) / kQTile, B * H);
        kern<<<grid, 256, smem, stream>>>(static_cast<const T*>(q), static_cast<const T*>(k),
                                         static_cast<const T*>(v), static_cast<T*>(y), N, w, scale);
        e = cudaGetLastError();
        if (e != cudaSuccess || k_cache == nullptr) return e;
        swa_fill_ring_kernel<T><<<B * H, 256, 0, stream>>>(static_cast<const T*>(k), static_cast<const T*>(v),
                                                          static_cast<T*>(k_cache), static_cast<T*>(v_cache), N, w);
        return cudaGetLastError();
    }
}

// bf16 decode, shared-memory variant (more heads than one wave of the register
// variant; bound by bytes in flight): 128 threads per (b, h). The valid slots of the head's key and
// value rings (slots 0..min(t, w-1)) are copied into shared memory with 16-byte
// asynchronous copies, so the data in flight costs no registers and many
// heads' copies are in flight per SM. Thread (warp, lane) owns the 16-byte
// piece c = lane % 8 (dims 8c..8c+7) of slots 16p + 4*warp + lane/8, p = 0..3,
// and copies that piece of the key and the value of its slots. Slots that
// neither this step (t) nor the previous one (t - 1) writes are copied before
// the wait for the previous kernel in the stream (griddepcontrol): only that
// kernel can still be running, and consecutive decode steps on one cache write
// slot (t - 1) mod w at most. Slot (t - 1) mod w is copied after the wait, and
// slot t mod w takes the new key and value (and is written back to the ring).
// Without `preload` (the ring was just written whole, by a prefill, or the
// kernel is launched in plain stream order) every slot is copied after the
// wait. The eight lanes of a slot combine their partial dot
// products by shuffles; every warp then reduces the 64 scores itself (max,
// exp, sum) from shared memory; the four warps' partial outputs are added
// through shared memory.
__global__ void __launch_bounds__(128)
swa_decode_bf16_smem_kernel(__nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc, long long t,
                       const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                       const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ y, int w, int new_slot,
                       float scale, int preload, unsigned* status) {
    __shared__ __align__(128) uint4 s_k[kMaxW * 8];      // slot rows of 128 bytes
    __shared__ __align__(128) uint4 s_v[kMaxW * 8];
    __shared__ float s_sc[kMaxW];
    __shared__ float s_part[4][kHead];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int c = lane & 7;
    const size_t bh = blockIdx.x;
    const size_t n_heads = gridDim.x;                    // extents of y and the ring for the index checks
    const int nvalid = t >= w ? w : (int)t + 1;          // slots holding a token: 0 .. nvalid-1
    const uint4* kring = reinterpret_cast<const uint4*>(kc + bh * w * kHead);
    const uint4* vring = reinterpret_cast<const uint4*>(vc + bh * w * kHead);
    const int prev_slot = new_slot == 0 ? w - 1 : new_slot - 1;
    auto copy_slot = [&](int slot) {
        cp_async16(tc::smem_u32(&s_k[slot * 8 + c]), kring + slot * 8 + c);
        cp_async16(tc::smem_u32(&s_v[slot * 8 + c]), vring + slot * 8 + c);
    };
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int slot = 16 * p + 4 * warp + (lane >> 3);
        if (preload && slot < nvalid && slot != new_slot && slot != prev_slot) copy_slot(slot);
    }
    grid_dependency_wait();
    const uint4 knew = __ldg(reinterpret_cast<const uint4*>(k + bh * kHead) + c);
    const uint4 vnew = __ldg(reinterpret_cast<const uint4*>(v + bh * kHead) + c);
    const uint4 qu = __ldg(reinterpret_cast<const uint4*>(q + bh * kHead) + c);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int slot = 16 * p + 4 * warp + (lane >> 3);
        if (slot >= nvalid) continue;
        if (slot == new_slot) {
            s_k[slot * 8 + c] = knew;
            s_v[slot * 8 + c] = vnew;
        } else if (!preload || slot == prev_slot) {
            copy_slot(slot);
        }
    }
    if (tid < 8 && in_bounds((bh * w + new_slot) * kHead + 8 * c + 7, n_heads * w * kHead, status)) {
        reinterpret_cast<uint4*>(kc + (bh * w + new_slot) * kHead)[c] = knew;
        reinterpret_cast<uint4*>(vc + (bh * w + new_slot) * kHead)[c] = vnew;
    }
    cp_async_wait_all();
    __syncthreads();
    // No early trigger for the next kernel: with more CTAs than one wave, its
    // CTAs would become resident and wait while this grid still has CTAs to run.
    float qv[8];
    {
        const uint32_t wd[4] = {qu.x, qu.y, qu.z, qu.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            qv[2 * e] = __uint_as_float(wd[e] << 16) * scale;
            qv[2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u) * scale;
        }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int slot = 16 * p + 4 * warp + (lane >> 3);
        const bool valid = slot < nvalid;
        const uint4 kr = valid ? s_k[slot * 8 + c] : make_uint4(0, 0, 0, 0);
        const uint32_t wd[4] = {kr.x, kr.y, kr.z, kr.w};
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            part = fmaf(qv[2 * e], __uint_as_float(wd[e] << 16), part);
            part = fmaf(qv[2 * e + 1], __uint_as_float(wd[e] & 0xFFFF0000u), part);
        }
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        part += __shfl_xor_sync(0xffffffffu, part, 4);
        if (c == 0) s_sc[slot] = valid ? part : -INFINITY;
    }
    __syncthreads();
    // Softmax statistics, computed by every warp (slot 0 always holds a token).
    const float a = s_sc[lane], bsc = s_sc[lane + 32];
    float m = fmaxf(a, bsc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = (a == -INFINITY ? 0.f : expf(a - m)) + (bsc == -INFINITY ? 0.f : expf(bsc - m));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.f / sum;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int slot = 16 * p + 4 * warp + (lane >> 3);
        if (slot >= nvalid) continue;
        const float pr = expf(s_sc[slot] - m) * inv;
        const uint4 vr = s_v[slot * 8 + c];
        const uint32_t wd[4] = {vr.x, vr.y, vr.z, vr.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[2 * e] = fmaf(pr, __uint_as_float(wd[e] << 16), acc[2 * e]);
            acc[2 * e + 1] = fmaf(pr, __uint_as_float(wd[e] & 0xFFFF0000u), acc[2 * e + 1]);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    }
    if (lane < 8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s_part[warp][8 * c + e] = acc[e];
    }
    __syncthreads();
    if (tid < 8) {
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            o[e] = s_part[0][8 * tid + e] + s_part[1][8 * tid + e] + s_part[2][8 * tid + e] + s_part[3][8 * tid + e];
        uint4 packed;
        packed.x = pack2(o[0], o[1]);
        packed.y = pack2(o[2], o[3]);
        packed.z = pack2(o[4], o[5]);
        packed.w = pack2(o[6], o[7]);
        if (in_bounds(bh * kHead + 8 * tid + 7, n_heads * kHead, status))
            reinterpret_cast<uint4*>(y + bh * kHead)[tid] = packed;
    }
}

// bf16 decode, register variant (used while every head's CTA fits one wave at
// eight CTAs per SM, where the step is bound by latency): 128 threads per
// (b, h), one memory round trip. Thread (warp,
// lane) owns the 16-byte piece c = lane % 8 (dims 8c..8c+7) of slots
// 16p + 4*warp + lane/8, p = 0..3, and loads that piece of both the key and the
// value of its four slots up front, together with q and the new key/value. The
// eight lanes of a slot combine their partial dot products by shuffles; every
// warp then reduces the 64 scores itself (max, exp, sum) from shared memory, so
// the weights are applied to values already in registers; the four warps'
// partial outputs are added through shared memory.
__global__ void __launch_bounds__(128)
swa_decode_bf16_reg_kernel(__nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc, long long t,
                       const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                       const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ y, int w, int new_slot,
                       float scale, int preload, unsigned* status) {
    __shared__ float s_sc[kMaxW];
    __shared__ float s_part[4][kHead];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int c = lane & 7;
    const size_t bh = blockIdx.x;

    // Slots that neither this step (t) nor the previous one (t - 1) writes are
    // loaded before the wait for the previous kernel in the stream: only that
    // kernel can still be running, and consecutive decode steps on one cache
    // write slot (t - 1) mod w at most. The rest is loaded after the wait.
    // Without `preload` (the ring was just written whole, by a prefill) every
    // slot is loaded after the wait.
    const int prev_slot = new_slot == 0 ? w - 1 : new_slot - 1;
    uint4 kr[4], vr[4];
    bool valid[4], late[4];
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int slot = 16 * p + 4 * warp + (lane >> 3);
        // newest token held by the slot: u = t - ((t - slot) mod w), empty while u < 0,
        // that is: every slot once t >= w, else the slots <= t.
        valid[p] = slot < w && (t >= w || slot <= t);
        late[p] = !preload || slot == new_slot || slot == prev_slot;
        kr[p] = vr[p] = make_uint4(0, 0, 0, 0);
        if (valid[p] && !late[p]) {
            kr[p] = __ldg(reinterpret_cast<const uint4*>(kc + (bh * w + slot) * kHead) + c);
            vr[p] = __ldg(reinterpret_cast<const uint4*>(vc + (bh * w + slot) * kHead) + c);
        }
    }
    grid_dependency_wait();
    const uint4 knew = __ldg(reinterpret_cast<const uint4*>(k + bh * kHead) + c);
    const uint4 vnew = __ldg(reinterpret_cast<const uint4*>(v + bh * kHead) + c);
    const uint4 qu = __ldg(reinterpret_cast<const uint4*>(q + bh * kHead) + c);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const int slot = 16 * p + 4 * warp + (lane >> 3);
        if (valid[p] && late[p]) {
            if (slot == new_slot) {
                kr[p] = knew;
                vr[p] = vnew;
            } else {
                kr[p] = reinterpret_cast<const uint4*>(kc + (bh * w + slot) * kHead)[c];
                vr[p] = reinterpret_cast<const uint4*>(vc + (bh * w + slot) * kHead)[c];
            }
        }
    }
    const size_t n_heads = gridDim.x;                // extents of y and the ring for the index checks
    if (tid < 8 && in_bounds((bh * w + new_slot) * kHead + 8 * c + 7, n_heads * w * kHead, status)) {
        reinterpret_cast<uint4*>(kc + (bh * w + new_slot) * kHead)[c] = knew;
        reinterpret_cast<uint4*>(vc + (bh * w + new_slot) * kHead)[c] = vnew;
    }
    grid_launch_dependents();           // the next step may be scheduled; it waits for this one to finish
    float qv[8];
    {
        const uint32_t wd[4] = {qu.x, qu.y, qu.z, qu.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            qv[2 * e] = __uint_as_float(wd[e] << 16) * scale;
            qv[2 * e + 1] = __uint_as_float(wd[e] & 0xFFFF0000u) * scale;
        }
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        const uint32_t wd[4] = {kr[p].x, kr[p].y, kr[p].z, kr[p].w};
        float part = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            part = fmaf(qv[2 * e], __uint_as_float(wd[e] << 16), part);
            part = fmaf(qv[2 * e + 1], __uint_as_float(wd[e] & 0xFFFF0000u), part);
        }
        part += __shfl_xor_sync(0xffffffffu, part, 1);
        part += __shfl_xor_sync(0xffffffffu, part, 2);
        part += __shfl_xor_sync(0xffffffffu, part, 4);
        if (c == 0) s_sc[16 * p + 4 * warp + (lane >> 3)] = valid[p] ? part : -INFINITY;
    }
    __syncthreads();
    // Softmax statistics, computed by every warp (slot 0 always holds a token).
    const float a = s_sc[lane], b = s_sc[lane + 32];
    float m = fmaxf(a, b);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float sum = (a == -INFINITY ? 0.f : expf(a - m)) + (b == -INFINITY ? 0.f : expf(b - m));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
    const float inv = 1.f / sum;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
        if (!valid[p]) continue;
        const float pr = expf(s_sc[16 * p + 4 * warp + (lane >> 3)] - m) * inv;
        const uint32_t wd[4] = {vr[p].x, vr[p].y, vr[p].z, vr[p].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            acc[2 * e] = fmaf(pr, __uint_as_float(wd[e] << 16), acc[2 * e]);
            acc[2 * e + 1] = fmaf(pr, __uint_as_float(wd[e] & 0xFFFF0000u), acc[2 * e + 1]);
        }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 8);
        acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], 16);
    }
    if (lane < 8) {
#pragma unroll
        for (int e = 0; e < 8; ++e) s_part[warp][8 * c + e] = acc[e];
    }
    __syncthreads();
    if (tid < 8) {
        float o[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            o[e] = s_part[0][8 * tid + e] + s_part[1][8 * tid + e] + s_part[2][8 * tid + e] + s_part[3][8 * tid + e];
        uint4 packed;
        packed.x = pack2(o[0], o[1]);
        packed.y = pack2(o[2], o[3]);
        packed.z = pack2(o[4], o[5]);
        packed.w = pack2(o[6], o[7]);
        if (in_bounds(bh * kHead + 8 * tid + 7, n_heads * kHead, status))
            reinterpret_cast<uint4*>(y + bh * kHead)[tid] = packed;
    }
}

}  // namespace

cudaError_t launch_swa_prefill(const void* q, const void* k, const void* v, void* y, void* k_cache,
                               void* v_cache, int B, int H, int N, int d, int w, float scale,
                               bool bf16, unsigned* status, unsigned debug, cudaStream_t stream) {
    if (d != kHead || w < 1 || w > kMaxW) return cudaErrorInvalidValue;
    return bf16 ? prefill_t<__nv_bfloat16>(q, k, v, y, k_cache, v_cache, B, H, N, w, scale, status, debug, stream)
                : prefill_t<float>(q, k, v, y, k_cache, v_cache, B, H, N, w, scale, status, debug, stream);
}

cudaError_t launch_swa_decode(void* k_cache, void* v_cache, int64_t t, const void* q, const void* k,
                              const void* v, void* y, int B, int H, int d, int w, float scale,
                              bool bf16, bool preload, int num_sms, unsigned* status, cudaStream_t stream) {
    if (d != kHead || w < 1 || w > kMaxW) return cudaErrorInvalidValue;
    if (bf16) {
        // Every head's CTA in one wave of the register variant (8 per SM): bound by
        // latency, where the register variant is quicker, launched as a
        // programmatic dependent (its CTAs are scheduled while the previous kernel
        // drains, and wait with griddepcontrol before reading what it wrote).
        // Beyond one wave the shared-memory variant keeps more bytes in flight; it
        // is launched in plain stream order, since CTAs that became resident early
        // and then waited would hold shared memory the previous kernel's last
        // CTAs need (every slot is then copied at once).
        const bool one_wave = (long long)B * H <= 8LL * num_sms;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(B * H));
        cfg.blockDim = dim3(128);
        cfg.stream = stream;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = one_wave ? 1 : 0;
        cudaError_t e = cudaLaunchKernelEx(&cfg, one_wave ? swa_decode_bf16_reg_kernel : swa_decode_bf16_smem_kernel,
                                           static_cast<__nv_bfloat16*>(k_cache),
                                           static_cast<__nv_bfloat16*>(v_cache), (long long)t,
                                           static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
                                           static_cast<const __nv_bfloat16*>(v), static_cast<__nv_bfloat16*>(y), w,
                                           (int)(t % w), scale, (preload && one_wave) ? 1 : 0, status);
        if (e != cudaSuccess) return e;
    } else {
        swa_decode_kernel<float><<<B * H, kMaxW, 0, stream>>>(
            static_cast<float*>(k_cache), static_cast<float*>(v_cache), (long long)t,
            static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
            static_cast<float*>(y), w, scale, status);
    }
    return cudaGetLastError();
}

}  // namespace based

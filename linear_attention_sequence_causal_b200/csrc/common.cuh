// Shared device helpers for the BASED kernels (sm_100a).
#pragma once

#include <utility>

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace based {

// Bits of the per-device status word (read and cleared by based_get_last_error).
enum : unsigned {
    DEV_ERR_TIMEOUT = 1u,   // a bounded wait expired
    DEV_ERR_BOUNDS = 2u,    // debug builds: a store's index fell outside its buffer
};

// Index check of a hand-indexed global store. In a build with
// BASED_DEBUG_BOUNDS defined (the debug library), an index outside [0, extent)
// records DEV_ERR_BOUNDS in the status word and the store is skipped; in the
// regular build it compiles to nothing.
__device__ __forceinline__ bool in_bounds(size_t idx, size_t extent, unsigned* status) {
#ifdef BASED_DEBUG_BOUNDS
    if (idx < extent) return true;
    if (status != nullptr) atomicOr(status, DEV_ERR_BOUNDS);
    return false;
#else
    (void)idx;
    (void)extent;
    (void)status;
    return true;
#endif
}

// Inputs are read as fp32 regardless of storage type.
__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Programmatic dependent launch (a grid launched with
// cudaLaunchAttributeProgrammaticStreamSerialization may start while the
// previous grid in the stream drains). grid_dependency_wait() returns once the
// grids this one depends on have completed and their writes are visible, and is
// a no-op without such a dependency; nothing produced by an earlier kernel may
// be read before it. grid_launch_dependents() lets the next such grid be
// scheduled early.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Host: launch `kernel` as a programmatic dependent of the previous work in
// `stream` (its CTAs may be scheduled while that work drains; the kernel calls
// grid_dependency_wait() before reading anything it produced).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Symmetric (packed) feature order: 0 is the constant, 1..d' are x_a, and
// 1 + d' + p for the p-th pair (a, b), a <= b, a-major, is x_a x_b (times
// 1/sqrt2 when a == b). packed_pair(p) returns (a, b) of pair p.
__host__ __device__ inline void packed_pair(int p, int d_feat, int& a, int& b) {
    a = 0;
    while (p >= d_feat - a) {
        p -= d_feat - a;
        ++a;
    }
    b = a + p;
}

// Global nanosecond timer, used to bound every spin wait.
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Upper bound of any single wait inside a kernel. A wait that runs past it
// records DEV_ERR_TIMEOUT and gives up; nothing ever spins without a bound.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

// sqrt(1/2) as an fp32 literal: the order-2 Taylor features carry 1/sqrt(2).
constexpr float kSqrtHalf = 0.70710678118654752440f;

__host__ __device__ constexpr int feature_dim(int d_feat) { return 1 + d_feat + d_feat * d_feat; }
// Distinct features of phi once the symmetric outer product is folded:
// 1 + d' + d'(d'+1)/2 (153 at d' = 16, 561 at d' = 32).
__host__ __device__ constexpr int sym_feature_dim(int d_feat) {
    return 1 + d_feat + d_feat * (d_feat + 1) / 2;
}

}  // namespace based

// C ABI of libbased: argument validation, kernel selection, device status word.
// The declarations and the contract of every entry point are in include/based.h.
#include <atomic>
#include <cstdint>
#include <cstdlib>
#include <mutex>

#include <cuda.h>

#include "../../include/based.h"
#include "common.cuh"
#include "kernels.h"

namespace {

// Per-device status word written by kernels whose bounded waits expired.
__device__ unsigned g_based_status;

constexpr int kMaxDevices = 64;
std::atomic<int> g_num_sms[kMaxDevices];

bool current_device(int* dev) { return cudaGetDevice(dev) == cudaSuccess && *dev >= 0 && *dev < kMaxDevices; }

// Unique id of the calling thread's current CUDA context (0 if unknown), from
// the driver through cudaGetDriverEntryPoint (the library does not link libcuda).
unsigned long long current_context_id() {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr ||
        get_id(ctx, &id) != CUDA_SUCCESS)
        return 0;
    return id;
}

// Device addresses of the library's __device__ symbols, per device and per
// context: cudaDeviceReset destroys the primary context with the module in it,
// and the next call runs in a new context where the symbol has a new address.
// A lookup is redone whenever the current context's id differs from the one
// the address was taken in.
struct SymbolSlot {
    const void* symbol;
    int dev;
    unsigned long long ctx;
    void* addr;
};
constexpr int kSymbolSlots = 4 * kMaxDevices;
std::mutex g_symbol_mu;
SymbolSlot g_symbols[kSymbolSlots];
int g_symbols_n = 0;

void* symbol_address(const void* symbol, int dev) {
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(g_symbol_mu);
    int slot = -1;
    for (int i = 0; i < g_symbols_n; ++i) {
        if (g_symbols[i].symbol == symbol && g_symbols[i].dev == dev) {
            if (ctx != 0 && g_symbols[i].ctx == ctx) return g_symbols[i].addr;
            slot = i;
            break;
        }
    }
    void* addr = nullptr;
    if (cudaGetSymbolAddress(&addr, symbol) != cudaSuccess || addr == nullptr) return nullptr;
    if (slot < 0) {
        if (g_symbols_n == kSymbolSlots) return addr;           // table full: no caching
        slot = g_symbols_n++;
    }
    g_symbols[slot] = SymbolSlot{symbol, dev, ctx, addr};
    return addr;
}

unsigned* status_word(int dev) { return static_cast<unsigned*>(symbol_address(&g_based_status, dev)); }

int num_sms(int dev) {
    int n = g_num_sms[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        g_num_sms[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// BASED_DEBUG_SKIP_MMA=1 in the environment makes the tensor-core kernels issue
// no MMA, so that their bounded waits expire: the failure-detection tests use it
// to check that a stalled kernel reports BASED_ERR_TIMEOUT and leaves the
// context usable. Read on every call; unset in normal use.
unsigned debug_flags() {
    const char* e = std::getenv("BASED_DEBUG_SKIP_MMA");
    return (e != nullptr && e[0] == '1') ? based::DEBUG_SKIP_MMA : 0u;
}

// Ring caches written whole by based_swa_prefill and not decoded from since.
// The first based_swa_decode on such a ring loads every slot after its
// dependency wait, because the prefill may be the kernel just before it in the
// stream and it writes every slot. Later steps read the slots that the step
// before them cannot write before the wait. The table keeps the most recent
// kFreshRings rings; a ring pushed out by that many later prefills of other
// rings is decoded as if no prefill had written it.
constexpr int kFreshRings = 256;
struct FreshRing { const void* cache; int dev; };
std::mutex g_fresh_mu;
FreshRing g_fresh[kFreshRings];
int g_fresh_n = 0;

void mark_ring_fresh(const void* cache, int dev) {
    std::lock_guard<std::mutex> lock(g_fresh_mu);
    for (int i = 0; i < g_fresh_n; ++i)
        if (g_fresh[i].cache == cache && g_fresh[i].dev == dev) return;
    if (g_fresh_n == kFreshRings) --g_fresh_n;                  // forget the oldest
    for (int i = g_fresh_n; i > 0; --i) g_fresh[i] = g_fresh[i - 1];
    g_fresh[0] = FreshRing{cache, dev};
    ++g_fresh_n;
}

// True (and the entry removed) when `cache` was written by a prefill since its last decode.
bool take_ring_fresh(const void* cache, int dev) {
    std::lock_guard<std::mutex> lock(g_fresh_mu);
    for (int i = 0; i < g_fresh_n; ++i) {
        if (g_fresh[i].cache == cache && g_fresh[i].dev == dev) {
            for (int j = i; j + 1 < g_fresh_n; ++j) g_fresh[j] = g_fresh[j + 1];
            --g_fresh_n;
            return true;
        }
    }
    return false;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }
bool ok_dtype(based_dtype_t d) { return d == BASED_F32 || d == BASED_BF16; }
bool la_dims_built(int d_feat, int d_v) {
    return (d_feat == 16 || d_feat == 32) && (d_v == 64 || d_v == 128);
}

// SIMT chunk sizes (shared memory bound: d' = 32 stops at 32 tokens).
bool simt_chunk_ok(int d_feat, int chunk) {
    return chunk == 16 || chunk == 32 || (chunk == 64 && d_feat == 16);
}

enum class LaPath { None, Simt, TensorCore, Quad };

// Kernel choice for a prefill. bf16: the chunked tcgen05 kernel where it is
// built (d' = 16, dv = 64; chunks of 64, 128 or 256 tokens, 128 by default),
// else the tcgen05 chunked quadratic path (any multiple of 128 tokens,
// kQuadDefaultChunk by default: the state of the other shapes does not fit one
// SM's tensor memory, so chunk start states go through the workspace); other
// explicit chunks (16, 32, and 64 for those shapes) and every fp32 call take
// the CUDA-core kernel.
LaPath choose_la_path(int d_feat, int d_v, based_dtype_t dtype, int* chunk) {
    const bool bf16 = dtype == BASED_BF16;
    if (*chunk == 0) {
        if (bf16 && based::la_prefill_tc_supported(d_feat, d_v, 128)) { *chunk = 128; return LaPath::TensorCore; }
        if (bf16 && based::la_prefill_quad_supported(d_feat, d_v)) {
            *chunk = based::kQuadDefaultChunk;
            return LaPath::Quad;
        }
        *chunk = d_feat == 16 ? 64 : 32;
        return LaPath::Simt;
    }
    if (bf16 && based::la_prefill_tc_supported(d_feat, d_v, *chunk)) return LaPath::TensorCore;
    if (bf16 && based::la_prefill_quad_supported(d_feat, d_v) && !based::la_prefill_tc_supported(d_feat, d_v, 128) &&
        based::la_prefill_quad_chunk_ok(*chunk))
        return LaPath::Quad;
    if (simt_chunk_ok(d_feat, *chunk)) return LaPath::Simt;
    return LaPath::None;
}

}  // namespace

namespace based {

// Lookups shared with the allocation-free prefill entry point (noalloc.cu).
unsigned* device_status_word(int dev) { return status_word(dev); }
void* device_symbol_address(const void* symbol, int dev) { return symbol_address(symbol, dev); }
int device_sm_count(int dev) { return num_sms(dev); }
unsigned current_debug_flags() { return debug_flags(); }
int resolve_la_path(int d_feat, int d_v, based_dtype_t dtype, int* chunk) {
    switch (choose_la_path(d_feat, d_v, dtype, chunk)) {
        case LaPath::Quad: return 3;
        case LaPath::TensorCore: return 2;
        case LaPath::Simt: return 1;
        default: return 0;
    }
}

}  // namespace based

extern "C" {

int based_version(void) { return 100; }

const char* based_status_string(based_status_t s) {
    switch (s) {
        case BASED_OK: return "BASED_OK";
        case BASED_ERR_INVALID_ARG: return "BASED_ERR_INVALID_ARG";
        case BASED_ERR_UNSUPPORTED: return "BASED_ERR_UNSUPPORTED";
        case BASED_ERR_CUDA: return "BASED_ERR_CUDA";
        case BASED_ERR_TIMEOUT: return "BASED_ERR_TIMEOUT";
        case BASED_ERR_BOUNDS: return "BASED_ERR_BOUNDS";
    }
    return "BASED_ERR_UNKNOWN";
}

size_t based_la_prefill_workspace(int B, int H, int N, int d_feat, int d_v, based_dtype_t dtype, int chunk) {
    if (B <= 0 || H <= 0 || N <= 0 || !ok_dtype(dtype) || !la_dims_built(d_feat, d_v)) return 0;
    int dev;
    if (!current_device(&dev)) return 0;
    const LaPath path = choose_la_path(d_feat, d_v, dtype, &chunk);
    if (path == LaPath::Quad) return based::la_prefill_quad_workspace(B, H, N, d_feat, d_v, chunk);
    if (path != LaPath::TensorCore) return 0;
    return based::la_prefill_tc_workspace(B, H, N, d_feat, d_v, chunk, num_sms(dev));
}

}  // extern "C"

namespace {

based_status_t la_prefill_impl(const void* q, const void* k, const void* v, void* y, float* S, float* z, int B,
                               int H, int N, int d_feat, int d_v, based_dtype_t dtype, int chunk, void* workspace,
                               size_t workspace_bytes, bool packed, cudaStream_t stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(y)) return BASED_ERR_INVALID_ARG;
    if ((S == nullptr) != (z == nullptr)) return BASED_ERR_INVALID_ARG;
    if (S != nullptr && (!aligned16(S) || !aligned16(z))) return BASED_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || chunk < 0 || !ok_dtype(dtype)) return BASED_ERR_INVALID_ARG;
    if (!la_dims_built(d_feat, d_v) || (long long)B * H > 65535) return BASED_ERR_UNSUPPORTED;
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    const int sms = num_sms(dev);
    unsigned* status = status_word(dev);
    if (sms <= 0 || status == nullptr) return BASED_ERR_CUDA;
    const LaPath path = choose_la_path(d_feat, d_v, dtype, &chunk);
    if (path == LaPath::None) return BASED_ERR_UNSUPPORTED;

    based::LaPrefillArgs a{q, k, v, y, S, z, B, H, N, d_feat, d_v, dtype == BASED_BF16, chunk,
                           workspace, workspace_bytes, status, debug_flags(), packed};
    cudaError_t e;
    if (path == LaPath::TensorCore) {
        const size_t need = based::la_prefill_tc_workspace(B, H, N, d_feat, d_v, chunk, sms);
        if (workspace_bytes < need || (need > 0 && !ok_ptr(workspace))) return BASED_ERR_INVALID_ARG;
        e = based::launch_la_prefill_tc(a, sms, stream);
    } else if (path == LaPath::Quad) {
        const size_t need = based::la_prefill_quad_workspace(B, H, N, d_feat, d_v, chunk);
        if (workspace_bytes < need || (need > 0 && !ok_ptr(workspace))) return BASED_ERR_INVALID_ARG;
        e = based::launch_la_prefill_quad(a, sms, stream);
    } else {
        e = based::launch_la_prefill_simt(a, stream);
    }
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

based_status_t la_decode_impl(float* S, float* z, const void* q, const void* k, const void* v, void* y,
                              const float* gamma, int B, int H, int d_feat, int d_v, based_dtype_t dtype,
                              bool packed, cudaStream_t stream) {
    if (!ok_ptr(S) || !ok_ptr(z) || !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(y))
        return BASED_ERR_INVALID_ARG;
    if (gamma != nullptr && (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0) return BASED_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || !ok_dtype(dtype)) return BASED_ERR_INVALID_ARG;
    if (!la_dims_built(d_feat, d_v) || (long long)B * H > (1LL << 30)) return BASED_ERR_UNSUPPORTED;
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    const int sms = num_sms(dev);
    unsigned* status = status_word(dev);
    if (sms <= 0 || status == nullptr) return BASED_ERR_CUDA;
    const cudaError_t e = based::launch_la_decode(S, z, q, k, v, y, gamma, B, H, d_feat, d_v, dtype == BASED_BF16,
                                                  packed, sms, status, stream);
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

}  // namespace

extern "C" {

based_status_t based_la_prefill(const void* q, const void* k, const void* v, void* y, float* S,
                                float* z, int B, int H, int N, int d_feat, int d_v,
                                based_dtype_t dtype, int chunk, void* workspace,
                                size_t workspace_bytes, cudaStream_t stream) {
    return la_prefill_impl(q, k, v, y, S, z, B, H, N, d_feat, d_v, dtype, chunk, workspace, workspace_bytes,
                           false, stream);
}

based_status_t based_la_prefill_packed(const void* q, const void* k, const void* v, void* y, float* S,
                                       float* z, int B, int H, int N, int d_feat, int d_v,
                                       based_dtype_t dtype, int chunk, void* workspace,
                                       size_t workspace_bytes, cudaStream_t stream) {
    return la_prefill_impl(q, k, v, y, S, z, B, H, N, d_feat, d_v, dtype, chunk, workspace, workspace_bytes,
                           true, stream);
}

size_t based_la_prefill_decay_workspace(int B, int H, int N, int d_feat, int d_v) {
    // (The bf16 paths; an fp32 call runs on the CUDA cores and needs none.)
    if (B <= 0 || H <= 0 || N <= 0 || !based::la_prefill_quad_supported(d_feat, d_v)) return 0;
    if (based::la_prefill_tc_supported(d_feat, d_v, 128)) {
        // The chunked kernel: segment totals, sized for this device's SMs.
        int dev;
        if (!current_device(&dev)) return 0;
        return based::la_prefill_tc_workspace(B, H, N, d_feat, d_v, 128, num_sms(dev));
    }
    return (size_t)B * H * ((N + 127) / 128) * sizeof(float);   // the quadratic form: log2 prefix of gamma
}

based_status_t based_la_prefill_decay(const void* q, const void* k, const void* v, void* y, float* S, float* z,
                                      const float* gamma, int B, int H, int N, int d_feat, int d_v,
                                      based_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(y)) return BASED_ERR_INVALID_ARG;
    if ((S == nullptr) != (z == nullptr)) return BASED_ERR_INVALID_ARG;
    if (S != nullptr && (!aligned16(S) || !aligned16(z))) return BASED_ERR_INVALID_ARG;
    if (gamma == nullptr || (reinterpret_cast<uintptr_t>(gamma) & 3u) != 0) return BASED_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || !ok_dtype(dtype)) return BASED_ERR_INVALID_ARG;
    if (!la_dims_built(d_feat, d_v) || (long long)B * H > 65535) return BASED_ERR_UNSUPPORTED;
    if (dtype == BASED_F32) {
        // fp32: the CUDA-core kernel, default chunk (64 tokens at d' = 16, 32 at d' = 32).
        int dev;
        if (!current_device(&dev)) return BASED_ERR_CUDA;
        unsigned* status = status_word(dev);
        if (status == nullptr) return BASED_ERR_CUDA;
        based::LaPrefillArgs a{q, k, v, y, S, z, B, H, N, d_feat, d_v, false, d_feat == 16 ? 64 : 32,
                               nullptr, 0, status, debug_flags(), false};
        a.gamma = gamma;
        const cudaError_t e = based::launch_la_prefill_simt(a, stream);
        return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
    }
    const bool chunked = based::la_prefill_tc_supported(d_feat, d_v, 128);
    if (!chunked) {
        const size_t need = (size_t)B * H * ((N + 127) / 128) * sizeof(float);
        if (workspace == nullptr || !aligned16(workspace) || workspace_bytes < need) return BASED_ERR_INVALID_ARG;
    }
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    const int sms = num_sms(dev);
    unsigned* status = status_word(dev);
    if (sms <= 0 || status == nullptr) return BASED_ERR_CUDA;
    if (chunked) {
        const size_t need = based::la_prefill_tc_workspace(B, H, N, d_feat, d_v, 128, sms);
        if (workspace_bytes < need || (need > 0 && !ok_ptr(workspace))) return BASED_ERR_INVALID_ARG;
    }
    based::LaPrefillArgs a{q, k, v, y, S, z, B, H, N, d_feat, d_v, true, 128, workspace, workspace_bytes,
                           status, debug_flags(), false};
    a.gamma = gamma;
    a.dlog = chunked ? nullptr : static_cast<float*>(workspace);
    // The chunked kernel where it is built (d' = 16, dv = 64), else the quadratic form.
    const cudaError_t e = chunked ? based::launch_la_prefill_tc(a, sms, stream) : based::launch_la_prefill_quad(a, sms, stream);
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

based_status_t based_la_decode_step(float* S, float* z, const void* q, const void* k, const void* v,
                                    void* y, int B, int H, int d_feat, int d_v, based_dtype_t dtype,
                                    cudaStream_t stream) {
    return la_decode_impl(S, z, q, k, v, y, nullptr, B, H, d_feat, d_v, dtype, false, stream);
}

based_status_t based_la_decode_step_packed(float* S, float* z, const void* q, const void* k, const void* v,
                                           void* y, int B, int H, int d_feat, int d_v, based_dtype_t dtype,
                                           cudaStream_t stream) {
    return la_decode_impl(S, z, q, k, v, y, nullptr, B, H, d_feat, d_v, dtype, true, stream);
}

based_status_t based_la_decode_step_decay(float* S, float* z, const void* q, const void* k, const void* v,
                                          void* y, const float* gamma, int B, int H, int d_feat, int d_v,
                                          based_dtype_t dtype, int packed, cudaStream_t stream) {
    if (gamma == nullptr) return BASED_ERR_INVALID_ARG;
    return la_decode_impl(S, z, q, k, v, y, gamma, B, H, d_feat, d_v, dtype, packed != 0, stream);
}

size_t based_la_backward_workspace(int B, int H, int N, int d_feat, int d_v, based_dtype_t dtype) {
    if (B <= 0 || H <= 0 || N <= 0 || dtype != BASED_BF16 || !based::la_backward_supported(d_feat, d_v)) return 0;
    return based::la_backward_workspace(B, H, N, d_feat, d_v);
}

based_status_t based_la_backward(const void* q, const void* k, const void* v, const void* y, const void* dy,
                                 void* dq, void* dk, void* dv, int B, int H, int N, int d_feat, int d_v,
                                 based_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(y) || !ok_ptr(dy)) return BASED_ERR_INVALID_ARG;
    if (!ok_ptr(dq) || !ok_ptr(dk) || !ok_ptr(dv)) return BASED_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || !ok_dtype(dtype)) return BASED_ERR_INVALID_ARG;
    if (dtype != BASED_BF16 || !based::la_backward_supported(d_feat, d_v)) return BASED_ERR_UNSUPPORTED;
    const long long tiles = (long long)B * H * ((N + 127) / 128);
    if (tiles > (1LL << 24)) return BASED_ERR_UNSUPPORTED;
    const size_t need = based::la_backward_workspace(B, H, N, d_feat, d_v);
    if (workspace == nullptr || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0 || workspace_bytes < need)
        return BASED_ERR_INVALID_ARG;
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    const int sms = num_sms(dev);
    unsigned* status = status_word(dev);
    if (sms <= 0 || status == nullptr) return BASED_ERR_CUDA;
    based::LaBackwardArgs a{q, k, v, y, dy, dq, dk, dv, B, H, N, d_feat, d_v, workspace, status, debug_flags()};
    const cudaError_t e = based::launch_la_backward(a, sms, stream);
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

based_status_t based_swa_prefill(const void* q, const void* k, const void* v, void* y, void* k_cache,
                                 void* v_cache, int B, int H, int N, int d, int w, float scale,
                                 based_dtype_t dtype, cudaStream_t stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(y)) return BASED_ERR_INVALID_ARG;
    if ((k_cache == nullptr) != (v_cache == nullptr)) return BASED_ERR_INVALID_ARG;
    if (k_cache != nullptr && (!aligned16(k_cache) || !aligned16(v_cache))) return BASED_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || w <= 0 || d <= 0 || !ok_dtype(dtype)) return BASED_ERR_INVALID_ARG;
    if (!(scale == scale) || scale - scale != 0.0f) return BASED_ERR_INVALID_ARG;   // NaN or inf
    if (d != 64 || w > 64 || (long long)B * H > 65535) return BASED_ERR_UNSUPPORTED;
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    unsigned* status = status_word(dev);
    if (status == nullptr) return BASED_ERR_CUDA;
    const cudaError_t e = based::launch_swa_prefill(q, k, v, y, k_cache, v_cache, B, H, N, d, w, scale,
                                                    dtype == BASED_BF16, status, debug_flags(), stream);
    if (e == cudaSuccess && k_cache != nullptr) mark_ring_fresh(k_cache, dev);
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

based_status_t based_swa_decode(void* k_cache, void* v_cache, int64_t t, const void* q, const void* k,
                                const void* v, void* y, int B, int H, int d, int w, float scale,
                                based_dtype_t dtype, cudaStream_t stream) {
    if (!ok_ptr(k_cache) || !ok_ptr(v_cache) || !ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(y))
        return BASED_ERR_INVALID_ARG;
    if (t < 0 || B <= 0 || H <= 0 || w <= 0 || d <= 0 || !ok_dtype(dtype)) return BASED_ERR_INVALID_ARG;
    if (!(scale == scale) || scale - scale != 0.0f) return BASED_ERR_INVALID_ARG;
    if (d != 64 || w > 64 || (long long)B * H > (1LL << 30)) return BASED_ERR_UNSUPPORTED;
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    unsigned* status = status_word(dev);
    if (status == nullptr) return BASED_ERR_CUDA;
    const bool preload = !take_ring_fresh(k_cache, dev);
    const cudaError_t e = based::launch_swa_decode(k_cache, v_cache, t, q, k, v, y, B, H, d, w, scale,
                                                   dtype == BASED_BF16, preload, num_sms(dev), status, stream);
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

based_status_t based_baseconv_prefill(const void* u_gate, const void* u_conv, const float* h,
                                      const float* bias, void* y, void* state, int B, int N, int d, int K,
                                      based_dtype_t dtype, cudaStream_t stream) {
    if (!ok_ptr(u_gate) || !ok_ptr(u_conv) || !ok_ptr(y)) return BASED_ERR_INVALID_ARG;
    if (!ok_ptr(h) || (bias != nullptr && !aligned16(bias))) return BASED_ERR_INVALID_ARG;
    if (state != nullptr && !aligned16(state)) return BASED_ERR_INVALID_ARG;
    if (B <= 0 || N <= 0 || d <= 0 || K <= 0 || !ok_dtype(dtype)) return BASED_ERR_INVALID_ARG;
    if (d % 4 != 0 || K > based::kMaxConvTaps || (long long)B * (d / 4) > (1LL << 30))
        return BASED_ERR_UNSUPPORTED;
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    const int sms = num_sms(dev);
    unsigned* status = status_word(dev);
    if (sms <= 0 || status == nullptr) return BASED_ERR_CUDA;
    const cudaError_t e = based::launch_baseconv_prefill(u_gate, u_conv, h, bias, y, state, B, N, d, K,
                                                         dtype == BASED_BF16, sms, status, stream);
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

based_status_t based_baseconv_decode(void* state, const void* u_gate, const void* u_conv, const float* h,
                                     const float* bias, void* y, int B, int d, int K, based_dtype_t dtype,
                                     cudaStream_t stream) {
    if (!ok_ptr(u_gate) || !ok_ptr(u_conv) || !ok_ptr(y)) return BASED_ERR_INVALID_ARG;
    if (!ok_ptr(h) || (bias != nullptr && !aligned16(bias))) return BASED_ERR_INVALID_ARG;
    if (K > 1 && !ok_ptr(state)) return BASED_ERR_INVALID_ARG;
    if (B <= 0 || d <= 0 || K <= 0 || !ok_dtype(dtype)) return BASED_ERR_INVALID_ARG;
    if (d % 4 != 0 || K > based::kMaxConvTaps || (long long)B * (d / 4) > (1LL << 30))
        return BASED_ERR_UNSUPPORTED;
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    unsigned* status = status_word(dev);
    if (status == nullptr) return BASED_ERR_CUDA;
    const cudaError_t e = based::launch_baseconv_decode(state, u_gate, u_conv, h, bias, y, B, d, K,
                                                        dtype == BASED_BF16, status, stream);
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

based_status_t based_get_last_error(cudaStream_t stream) {
    if (cudaStreamSynchronize(stream) != cudaSuccess) return BASED_ERR_CUDA;
    int dev;
    if (!current_device(&dev)) return BASED_ERR_CUDA;
    unsigned* status = status_word(dev);
    if (status == nullptr) return BASED_ERR_CUDA;
    unsigned word = 0;
    if (cudaMemcpy(&word, status, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return BASED_ERR_CUDA;
    if (word != 0) {
        const unsigned zero = 0;
        if (cudaMemcpy(status, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return BASED_ERR_CUDA;
    }
    if (word & based::DEV_ERR_TIMEOUT) return BASED_ERR_TIMEOUT;
    return (word & based::DEV_ERR_BOUNDS) ? BASED_ERR_BOUNDS : BASED_OK;
}

}  // extern "C"

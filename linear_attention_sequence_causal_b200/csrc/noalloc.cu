// based_la_prefill_noalloc: the linear-attention prefill for callers that may
// not allocate device memory themselves (see include/based.h). The segment
// totals that based_la_prefill keeps in a caller-provided workspace live here
// in a fixed array that is part of the library's device image.
#include "../../include/based.h"
#include "common.cuh"
#include "kernels.h"

namespace based {
unsigned* device_status_word(int dev);
void* device_symbol_address(const void* symbol, int dev);   // per device and CUDA context
int device_sm_count(int dev);
unsigned current_debug_flags();
int resolve_la_path(int d_feat, int d_v, based_dtype_t dtype, int* chunk);   // 0 none, 1 CUDA cores, 2 chunked tcgen05, 3 quadratic tcgen05
}  // namespace based

namespace {

// Largest scratch the prefill needs at the least: segment totals of at most one
// CTA per SM (148 x 160 x 80 fp32 = 7.6 MB on a B200), rounded up to 8 MiB. (The
// chunked kernel splits each total into pieces when its scratch has room for
// them; with this array it takes as many as fit.) Every GPU that loads the
// library holds this array until the process exits.
constexpr size_t kScratchBytes = size_t(8) << 20;
static __device__ __align__(256) unsigned char g_prefill_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_prefill_scratch on device `dev` (which must be current).
// The symbol's name in host code is only a stand-in; its device address is
// looked up on the first call in each CUDA context of the device (again after
// a cudaDeviceReset, which gives the device a new context and module).
void* scratch_address(int dev) { return based::device_symbol_address(&g_prefill_scratch, dev); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ok_ptr(const void* p) { return p != nullptr && aligned16(p); }

}  // namespace

extern "C" based_status_t based_la_prefill_noalloc(const void* q, const void* k, const void* v, void* y,
                                                   float* S, float* z, int B, int H, int N, int d_feat,
                                                   int d_v, based_dtype_t dtype, int chunk,
                                                   cudaStream_t stream) {
    if (!ok_ptr(q) || !ok_ptr(k) || !ok_ptr(v) || !ok_ptr(y)) return BASED_ERR_INVALID_ARG;
    if ((S == nullptr) != (z == nullptr)) return BASED_ERR_INVALID_ARG;
    if (S != nullptr && (!aligned16(S) || !aligned16(z))) return BASED_ERR_INVALID_ARG;
    if (B <= 0 || H <= 0 || N <= 0 || chunk < 0) return BASED_ERR_INVALID_ARG;
    if (dtype != BASED_F32 && dtype != BASED_BF16) return BASED_ERR_INVALID_ARG;
    if (!((d_feat == 16 || d_feat == 32) && (d_v == 64 || d_v == 128)) || (long long)B * H > 65535)
        return BASED_ERR_UNSUPPORTED;
    int dev;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return BASED_ERR_CUDA;
    const int sms = based::device_sm_count(dev);
    unsigned* status = based::device_status_word(dev);
    if (sms <= 0 || status == nullptr) return BASED_ERR_CUDA;
    const bool library_chunk = chunk == 0;
    const int path = based::resolve_la_path(d_feat, d_v, dtype, &chunk);
    if (path == 0) return BASED_ERR_UNSUPPORTED;
    size_t need = path == 2 ? based::la_prefill_tc_workspace_min(B, H, N, d_feat, d_v, chunk, sms)
                : path == 3 ? based::la_prefill_quad_workspace(B, H, N, d_feat, d_v, chunk)
                            : 0;
    if (path == 3 && need > kScratchBytes && library_chunk) {
        chunk = 0;          // the library's choice: one chunk (the quadratic form) needs no scratch
        need = 0;
    }
    if (need > kScratchBytes) return BASED_ERR_UNSUPPORTED;         // beyond the fixed scratch
    void* scratch = scratch_address(dev);
    if (scratch == nullptr) return BASED_ERR_CUDA;
    based::LaPrefillArgs a{q, k, v, y, S, z, B, H, N, d_feat, d_v, dtype == BASED_BF16, chunk,
                           scratch, kScratchBytes, status, based::current_debug_flags()};
    const cudaError_t e = path == 2   ? based::launch_la_prefill_tc(a, sms, stream)
                          : path == 3 ? based::launch_la_prefill_quad(a, sms, stream)
                                      : based::launch_la_prefill_simt(a, stream);
    return e == cudaSuccess ? BASED_OK : BASED_ERR_CUDA;
}

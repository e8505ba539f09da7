// Host-side launchers of the BASED kernels (internal to libbased; not part of the C ABI).
// Every launcher only enqueues work on `stream` and returns the launch's cudaError_t.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace based {

struct LaPrefillArgs {
    const void* q; const void* k; const void* v; void* y;
    float* S; float* z;              // may both be null
    int B, H, N, d_feat, d_v;
    bool bf16;
    int chunk;                       // resolved, never 0
    void* workspace; size_t ws_bytes;
    unsigned* status;                // device status word
    unsigned debug;                  // DEBUG_* bits (testing only)
    bool packed = false;             // final state in the symmetric layout (1 + d' + d'(d'+1)/2 rows)
    const float* gamma = nullptr;    // coarse decay: [B*H][ceil(N/128)] per 128-token tile (quadratic path)
    float* dlog = nullptr;           // with gamma: [B*H][ceil(N/128)] fp32 scratch for its log2 prefix
};

// Testing aid: with this bit the tensor-core kernels issue no MMA, so their
// bounded waits expire and report DEV_ERR_TIMEOUT (see debug_flags() in api.cu).
constexpr unsigned DEBUG_SKIP_MMA = 1u;

// SIMT fp32-arithmetic path: any supported dtype, chunk in {16, 32, 64}.
cudaError_t launch_la_prefill_simt(const LaPrefillArgs& a, cudaStream_t stream);

// Tensor-core (tcgen05/TMEM) path: bf16 inputs, d' = 16, dv = 64, chunk = 128.
bool la_prefill_tc_supported(int d_feat, int d_v, int chunk);
// Workspace for the segment totals: the size that lets the totals pass split
// every total into the pieces that fill the SMs best, and the least it can run
// with (one piece per total); the launcher splits as finely as ws_bytes allows.
size_t la_prefill_tc_workspace(int B, int H, int N, int d_feat, int d_v, int chunk, int num_sms);
size_t la_prefill_tc_workspace_min(int B, int H, int N, int d_feat, int d_v, int chunk, int num_sms);
cudaError_t launch_la_prefill_tc(const LaPrefillArgs& a, int num_sms, cudaStream_t stream);

// Tensor-core chunked path for the shapes whose state does not fit one SM's
// tensor memory (bf16, any built d', dv): the start state of every chunk by a
// sweep over the tokens (into the workspace), then y from the masked quadratic
// form within each chunk plus phi(q) against its chunk's start state. chunk: a
// multiple of 128 tokens; 0 (LaPrefillArgs) or >= N: one chunk, the plain
// quadratic form, no workspace.
bool la_prefill_quad_supported(int d_feat, int d_v);
bool la_prefill_quad_chunk_ok(int chunk);
size_t la_prefill_quad_workspace(int B, int H, int N, int d_feat, int d_v, int chunk);
cudaError_t launch_la_prefill_quad(const LaPrefillArgs& a, int num_sms, cudaStream_t stream);
// Chunk of the chunked quadratic path when the caller leaves the choice to the library.
constexpr int kQuadDefaultChunk = 1024;

// Backward (training) pass of the causal Taylor linear attention, bf16 tensor
// cores: dq, dk, dv from q, k, v, the forward's y and the upstream dy.
struct LaBackwardArgs {
    const void* q; const void* k; const void* v; const void* y; const void* dy;
    void* dq; void* dk; void* dv;
    int B, H, N, d_feat, d_v;
    void* workspace;                 // >= la_backward_workspace(B, H, N, d_feat, d_v) bytes, 256-byte aligned
    unsigned* status;
    unsigned debug;
};
bool la_backward_supported(int d_feat, int d_v);
size_t la_backward_workspace(int B, int H, int N, int d_feat, int d_v);
size_t la_backward_g_bytes(const LaBackwardArgs& a);
cudaError_t launch_la_backward(const LaBackwardArgs& a, int num_sms, cudaStream_t stream);

// `packed`: S and z hold the symmetric layout (1 + d' + d'(d'+1)/2 rows).
// gamma: [B, H] fp32 decay applied to S, z before the token (nullptr: none).
cudaError_t launch_la_decode(float* S, float* z, const void* q, const void* k, const void* v,
                             void* y, const float* gamma, int B, int H, int d_feat, int d_v, bool bf16,
                             bool packed, int num_sms, unsigned* status, cudaStream_t stream);

cudaError_t launch_swa_prefill(const void* q, const void* k, const void* v, void* y,
                               void* k_cache, void* v_cache, int B, int H, int N, int d, int w,
                               float scale, bool bf16, unsigned* status, unsigned debug,
                               cudaStream_t stream);

// Tensor-core path of the sliding-window prefill (bf16, d = 64, w <= 64), ring fill fused.
cudaError_t launch_swa_prefill_tc(const void* q, const void* k, const void* v, void* y, void* k_cache,
                                  void* v_cache, int B, int H, int N, int w, float scale, unsigned* status,
                                  unsigned debug, cudaStream_t stream);

// preload: the bf16 kernel may read the ring slots other than t mod w and
// (t-1) mod w before its dependency wait (see based_swa_decode in based.h);
// false when the kernel before it may have written any slot of this ring.
cudaError_t launch_swa_decode(void* k_cache, void* v_cache, int64_t t, const void* q,
                              const void* k, const void* v, void* y, int B, int H, int d, int w,
                              float scale, bool bf16, bool preload, int num_sms, unsigned* status,
                              cudaStream_t stream);

// Short gated convolution: filter taps K in [1, kMaxConvTaps], d a multiple of 4.
constexpr int kMaxConvTaps = 8;
cudaError_t launch_baseconv_prefill(const void* gate, const void* conv, const float* h, const float* bias,
                                    void* y, void* state, int B, int N, int d, int K, bool bf16, int num_sms,
                                    unsigned* status, cudaStream_t stream);
cudaError_t launch_baseconv_decode(void* state, const void* gate, const void* conv, const float* h,
                                   const float* bias, void* y, int B, int d, int K, bool bf16,
                                   unsigned* status, cudaStream_t stream);

}  // namespace based

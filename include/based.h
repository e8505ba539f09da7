/*
 * based.h -- C ABI of the B200 (sm_100a) BASED hot path: causal Taylor linear
 * attention and sliding-window softmax attention, prefill and decode, plus the
 * short gated convolution (BaseConv) mixer.
 *
 * The method is that of "Simple linear attention language models balance the
 * recall-throughput tradeoff" (BASED, arXiv 2402.18668v2):
 *   - linear attention through a feature map, computed in a parallel form for
 *     prompt processing and a recurrent form for generation (§2 "Efficient
 *     attentions", §5 "Execution stages");
 *   - the 2nd-order Taylor feature map with projected dimension d' (§4 "Taylor
 *     Linear Attention"), used here in its explicit form
 *         phi(x) = [1, x, vec(x (x) x)/sqrt(2)],  D = 1 + d' + d'^2 features,
 *     so that phi(q).phi(k) = 1 + q.k + (q.k)^2/2;
 *   - outputs normalised by the "K-state" z (App. D.4 "State size");
 *   - exact softmax attention inside a small sliding window with a w-sized KV
 *     cache (§4 "Local Exact Attention");
 *   - short gated convolutions beside the window layers (§4, Additional
 *     mixers; App. C "Extended Architecture Details", Convolution).
 *
 * Conventions shared by every call
 * --------------------------------
 * - All tensors are dense, contiguous, row-major, batch-major then head-major,
 *   and live in device memory of the current CUDA device. Every pointer must
 *   be 16-byte aligned. The library never allocates memory and keeps no
 *   pointer after a call returns; the caller owns every buffer.
 * - dtype selects the element type of q, k, v, y, the SWA caches and the
 *   convolution's streams and state: BASED_F32 (float) or BASED_BF16
 *   (__nv_bfloat16). S, z and the convolution's taps and bias are always float.
 *   Arithmetic is fp32 (fp32 accumulation of bf16 tensor-core products on the
 *   bf16 prefill path).
 * - Work is enqueued on `stream` (0 = legacy default stream); every call is
 *   asynchronous. Argument errors are reported synchronously by the return
 *   value and enqueue nothing. Errors detected on the device (a bounded
 *   internal wait that expired) are recorded in a per-device status word read
 *   by based_get_last_error().
 * - Causality is inclusive: token i attends to keys j <= i.
 * - Feature order of phi and of the rows of S and z: index 0 is the constant
 *   1; 1..d' hold x_a; 1 + d' + a*d' + b holds x_a*x_b/sqrt(2).
 */
#ifndef BASED_H
#define BASED_H

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define BASED_API __attribute__((visibility("default")))
#else
#define BASED_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    BASED_OK = 0,
    BASED_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad size, workspace too small */
    BASED_ERR_UNSUPPORTED = 2,   /* valid but not built: d', dv, d, w, chunk or dtype outside the set */
    BASED_ERR_CUDA = 3,          /* a CUDA runtime call failed (launch, device query, sync) */
    BASED_ERR_TIMEOUT = 4,       /* a bounded wait inside a kernel expired; outputs are undefined */
    BASED_ERR_BOUNDS = 5         /* debug library only (built with BASED_DEBUG_BOUNDS): a kernel
                                    computed a store index outside its buffer; the store was
                                    skipped and the outputs are undefined */
} based_status_t;

typedef enum {
    BASED_F32 = 0,
    BASED_BF16 = 1
} based_dtype_t;

/*
 * based_la_prefill -- parallel (prompt-processing) form of causal Taylor linear
 * attention over N tokens, starting from an empty state.
 *
 * Computes, for every batch b, head h and token i,
 *     y_i = sum_{j<=i} a_ij v_j / sum_{j<=i} a_ij,   a_ij = 1 + q_i.k_j + (q_i.k_j)^2/2
 *         = phi(q_i)^T S_i / phi(q_i)^T z_i,         S_i = sum_{j<=i} phi(k_j) v_j^T,
 * and writes the final state S = S_{N-1} and z = z_{N-1}.
 * BASED §4 "Taylor Linear Attention"; App. B "Forward / Generation Prefill"
 * (Algorithm 1: y = T0 + T1 + T2, on-diagonal quadratic tiles with a local causal
 * mask plus an off-diagonal cumulative state); App. D.4 (K-state z).
 *
 *   q, k    [B, H, N, d_feat]  dtype, read only
 *   v       [B, H, N, d_v]     dtype, read only
 *   y       [B, H, N, d_v]     dtype, written (round-to-nearest for bf16)
 *   S       [B, H, D, d_v]     float, written; D = 1 + d_feat + d_feat^2
 *   z       [B, H, D]          float, written
 *           S and z may both be NULL (final state not wanted), not just one.
 *   d_feat  16 or 32;  d_v  64 or 128;  N >= 1;  B, H >= 1
 *   chunk   tokens per chunk (on-diagonal tile): 0 (library's choice) or one
 *           of the values built for the call. BASED_BF16 at d_feat 16, d_v 64:
 *           64, 128 or 256 on the tensor cores, the chunked form with the state
 *           in tensor memory (0 picks 128). BASED_BF16, other shapes (whose
 *           state does not fit one SM's tensor memory): any multiple of 128 on
 *           the tensor cores; the start state of every chunk is computed first
 *           into the workspace, then each chunk's outputs from the masked
 *           quadratic form within the chunk plus phi(q) against that state (0
 *           picks 1024; a chunk of at least N is the plain quadratic form and
 *           needs no workspace). Both dtypes: 16, 32 (and 64 at d_feat 16 for
 *           BASED_F32) on the CUDA cores in fp32 arithmetic (0 picks the
 *           largest for fp32). Other values return BASED_ERR_UNSUPPORTED. The
 *           result does not depend on the chunk beyond rounding.
 *   workspace, workspace_bytes
 *           device scratch of at least based_la_prefill_workspace(...) bytes
 *           (NULL allowed when that size is 0). Holds the chunk start states
 *           of the shapes whose state does not fit tensor memory (bf16, (d_feat
 *           x d_v) x (chunks - 1) x 128-feature tiles), or the segment totals
 *           that let long sequences of the d_feat 16, d_v 64 kernel run in
 *           segments at once (overwritten in place by the state entering each
 *           segment); its contents on entry do not matter.
 * Returns BASED_ERR_INVALID_ARG for null or misaligned pointers, non-positive
 * sizes, or a workspace smaller than required; BASED_ERR_UNSUPPORTED for a
 * (d_feat, d_v, dtype, chunk) combination outside the built set.
 */
BASED_API based_status_t based_la_prefill(const void* q, const void* k, const void* v, void* y,
                                float* S, float* z,
                                int B, int H, int N, int d_feat, int d_v,
                                based_dtype_t dtype, int chunk,
                                void* workspace, size_t workspace_bytes,
                                cudaStream_t stream);

/*
 * based_la_prefill_workspace -- bytes of device scratch based_la_prefill needs
 * for these arguments on the current device (0 when the call needs none: one
 * segment per sequence on the d_feat 16, d_v 64 kernel, one chunk on the
 * others, or the CUDA-core path).
 * Returns 0 for arguments based_la_prefill would reject.
 */
BASED_API size_t based_la_prefill_workspace(int B, int H, int N, int d_feat, int d_v,
                                  based_dtype_t dtype, int chunk);

/*
 * based_la_prefill_noalloc -- the same prefill as based_la_prefill, for callers
 * that cannot allocate device memory themselves: code running inside a memory
 * manager that owns every device buffer (a framework's caching allocator, a
 * serving runtime with a fixed pool, a plugin host that hands out only its own
 * tensors), or code on a latency-critical path where an allocation would stall
 * the device. It takes no workspace: the segment totals live in one fixed
 * 8 MiB array inside the library's device image, which every GPU that loads the
 * library keeps until the process exits. The paper has no counterpart; this is
 * a service of this library.
 *
 * Arguments, results and errors are those of based_la_prefill, minus the
 * workspace. It calls no cudaMalloc, cudaFree or other allocating routine. It
 * returns BASED_ERR_UNSUPPORTED when the call would need more scratch than the
 * fixed array holds (not the case on a B200 for the shapes this library builds).
 *
 * The first call on a device looks up the array's device address with that
 * device current, once per device; make that first call before any stream
 * capture. All calls share the one array, which keeps the last call's contents
 * (nothing in it needs to start at zero): calls that overlap on the GPU, for
 * example on two streams at once, race on it and must be serialised by the caller.
 */
BASED_API based_status_t based_la_prefill_noalloc(const void* q, const void* k, const void* v, void* y,
                                                  float* S, float* z,
                                                  int B, int H, int N, int d_feat, int d_v,
                                                  based_dtype_t dtype, int chunk,
                                                  cudaStream_t stream);

/*
 * based_la_decode_step -- recurrent (next-token) form: one generated token per
 * sequence. In place, for every (b, h):
 *     S += phi(k) v^T;  z += phi(k);  y = phi(q)^T S / phi(q)^T z
 * (the output includes the current token). BASED §2 "Efficient attentions"
 * (recurrent generation), App. B "Next Token Prediction" (KV-state update).
 *
 *   S       [B, H, D, d_v] float, read and written in place
 *   z       [B, H, D]      float, read and written in place
 *   q, k    [B, H, d_feat] dtype;  v [B, H, d_v] dtype
 *   y       [B, H, d_v]    dtype, written
 *   d_feat  16 or 32;  d_v 64 or 128
 * A state produced by based_la_prefill over N tokens followed by M decode steps
 * equals, up to rounding, the state of a prefill over N + M tokens.
 */
BASED_API based_status_t based_la_decode_step(float* S, float* z,
                                    const void* q, const void* k, const void* v, void* y,
                                    int B, int H, int d_feat, int d_v,
                                    based_dtype_t dtype, cudaStream_t stream);

/*
 * Symmetric (packed) state layout -- an extension of this library, not a form
 * the pages print. The order-2 block of phi is the symmetric outer product
 * x (x) x, so the state needs only one row per unordered pair (a, b):
 *     phi_s(x) = [1, x, x_a x_b for a <= b (a-major), times 1/sqrt2 when a == b],
 * D_s = 1 + d_feat + d_feat (d_feat + 1) / 2 rows (153 at d_feat 16, 561 at 32),
 * with phi_s(q).phi_s(k) = phi(q).phi(k) = 1 + q.k + (q.k)^2/2 (derived from
 * BASED §4 "Taylor Linear Attention"). Row order: 0 the constant, 1..d_feat
 * the x_a, then 1 + d_feat + p for the p-th pair (a, b) in the order
 * (0,0), (0,1), .., (0,d_feat-1), (1,1), .., (d_feat-1,d_feat-1). In terms of
 * the full layout, packed row (a, b) equals full row (a, a) when a == b and
 * (full (a, b) + full (b, a)) / sqrt2 when a < b. Decode reads and writes
 * ~44 % fewer state bytes per token in this layout.
 */

/*
 * based_la_prefill_packed -- based_la_prefill, writing the final state in the
 * symmetric layout: S [B, H, D_s, d_v] and z [B, H, D_s] (float). Arguments,
 * workspace (based_la_prefill_workspace gives its size), results for y, and
 * errors are those of based_la_prefill.
 */
BASED_API based_status_t based_la_prefill_packed(const void* q, const void* k, const void* v, void* y,
                                                 float* S, float* z,
                                                 int B, int H, int N, int d_feat, int d_v,
                                                 based_dtype_t dtype, int chunk,
                                                 void* workspace, size_t workspace_bytes,
                                                 cudaStream_t stream);

/*
 * based_la_decode_step_packed -- based_la_decode_step on a state in the
 * symmetric layout: S [B, H, D_s, d_v] and z [B, H, D_s], read and written in
 * place. Arguments, results and errors are otherwise those of
 * based_la_decode_step.
 */
BASED_API based_status_t based_la_decode_step_packed(float* S, float* z,
                                                     const void* q, const void* k, const void* v, void* y,
                                                     int B, int H, int d_feat, int d_v,
                                                     based_dtype_t dtype, cudaStream_t stream);

/*
 * Coarse input-dependent decay (BASED App. C "Extended Architecture Details",
 * Decay; App. D.4 "BASED Quality Ablations"). The pages print no formula; the
 * reading implemented: one scalar gamma per 128-token tile scales the state
 * where the tile begins, S_c = gamma_c S_{c-1} + sum_{t in tile c} phi(k_t) v_t^T
 * (z likewise), and a tile's own keys are not decayed among themselves. Key j
 * reaches query i >= j with the weight prod_{c = tile(j)+1 .. tile(i)} gamma_c,
 * in the numerator and the denominator alike. gamma values lie in (0, 1].
 *
 * based_la_prefill_decay -- based_la_prefill with decay: gamma [B, H,
 * ceil(N/128)] fp32 (device), one value per tile (tile 0's is unused).
 * d_feat in {16, 32}, d_v in {64, 128}, else BASED_ERR_UNSUPPORTED. bf16 runs
 * on the tensor cores (the chunked kernel at d_feat 16 / d_v 64, the quadratic
 * form otherwise), fp32 on the CUDA cores (no workspace). S and z (optional
 * together, full 1 + d' + d'^2 layout) receive the decayed final state.
 * workspace >= based_la_prefill_decay_workspace(B, H, N, d_feat, d_v) bytes of
 * device memory, 16-byte aligned (segment totals of the chunked kernel, or the
 * per-tile log2 prefix sums of gamma; the chunked kernel's size depends on the
 * current device's SM count, and may be 0).
 */
BASED_API size_t based_la_prefill_decay_workspace(int B, int H, int N, int d_feat, int d_v);
BASED_API based_status_t based_la_prefill_decay(const void* q, const void* k, const void* v, void* y,
                                                float* S, float* z, const float* gamma,
                                                int B, int H, int N, int d_feat, int d_v,
                                                based_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                                cudaStream_t stream);

/*
 * based_la_decode_step_decay -- based_la_decode_step (packed = 0) or
 * based_la_decode_step_packed (packed = 1) with the state first scaled by
 * gamma [B, H] fp32 (device): S <- gamma S, z <- gamma z, then the token's
 * update and output. Pass the tile's gamma on the first token of a 128-token
 * tile and 1 otherwise to continue a decayed prefill. Errors as the undecayed
 * step; gamma NULL returns BASED_ERR_INVALID_ARG.
 */
BASED_API based_status_t based_la_decode_step_decay(float* S, float* z, const void* q, const void* k,
                                                    const void* v, void* y, const float* gamma,
                                                    int B, int H, int d_feat, int d_v,
                                                    based_dtype_t dtype, int packed, cudaStream_t stream);

/*
 * based_la_backward -- gradients of the causal Taylor linear attention of
 * based_la_prefill (the training form of the prefill stage, BASED §5
 * "Execution stages"). With s_ij = q_i.k_j, a_ij = 1 + s_ij + s_ij^2/2,
 * den_i = sum_{j<=i} a_ij and the forward's output y, for an upstream
 * gradient dy:
 *     g_i = dy_i / den_i,   c_i = g_i . y_i,
 *     ds_ij = (g_i . v_j - c_i)(1 + s_ij)   for j <= i (0 otherwise),
 *     dq_i = sum_j ds_ij k_j,   dk_j = sum_i ds_ij q_i,   dv_j = sum_i a_ij g_i.
 * These are the derivatives of y_i = sum_{j<=i} a_ij v_j / den_i, the exact
 * quadratic form of the feature map of §4 "Taylor Linear Attention".
 *
 *   q, k      [B, H, N, d_feat] bf16      (the prefill's inputs)
 *   v         [B, H, N, d_v] bf16
 *   y         [B, H, N, d_v] bf16         (the prefill's output for q, k, v)
 *   dy        [B, H, N, d_v] bf16         upstream gradient
 *   dq, dk    [B, H, N, d_feat] bf16      written
 *   dv        [B, H, N, d_v] bf16         written
 *   workspace >= based_la_backward_workspace(...) bytes of device memory,
 *             256-byte aligned; caller-owned, scratch for the call (g as bf16
 *             and c as fp32 per token, rows padded to a multiple of 128).
 * All pointers are device memory, 16-byte aligned, contiguous row-major, owned
 * by the caller; outputs must not alias inputs. Built for bf16 with
 * d_feat in {16, 32} and d_v in {64, 128}; fp32 and other sizes return
 * BASED_ERR_UNSUPPORTED. Three kernels are queued on `stream` (asynchronous);
 * BASED_ERR_TIMEOUT from based_get_last_error means a bounded wait expired and
 * the outputs are undefined.
 */
BASED_API size_t based_la_backward_workspace(int B, int H, int N, int d_feat, int d_v, based_dtype_t dtype);
BASED_API based_status_t based_la_backward(const void* q, const void* k, const void* v, const void* y,
                                           const void* dy, void* dq, void* dk, void* dv,
                                           int B, int H, int N, int d_feat, int d_v,
                                           based_dtype_t dtype, void* workspace, size_t workspace_bytes,
                                           cudaStream_t stream);

/*
 * based_swa_prefill -- causal sliding-window softmax attention over N tokens:
 *     y_i = sum_j softmax_j(scale * q_i.k_j) v_j  over  i - w < j <= i
 * (w keys including the query's own position). BASED §4 "Local Exact
 * Attention", App. A.1 (O(Nw) cost), App. C (TCWINDOW layers).
 *
 *   q, k, v, y  [B, H, N, d] dtype
 *   k_cache, v_cache  [B, H, w, d] dtype, written with the ring state after the
 *           prompt: slot t mod w holds token t for t in [max(0, N-w), N); slots
 *           never written are set to zero. Both NULL to skip.
 *   d 64;  1 <= w <= 64;  scale finite (the workloads use 1/sqrt(d))
 */
BASED_API based_status_t based_swa_prefill(const void* q, const void* k, const void* v, void* y,
                                 void* k_cache, void* v_cache,
                                 int B, int H, int N, int d, int w, float scale,
                                 based_dtype_t dtype, cudaStream_t stream);

/*
 * based_swa_decode -- one generated token per sequence over the w-slot ring
 * KV cache (BASED §4 "Local Exact Attention": a w-sized KV cache; App. B
 * "Next Token Prediction"). t is the number of tokens every sequence has seen
 * before this one. Writes (k, v) into slot t mod w, then attends over the
 * min(t+1, w) slots holding tokens max(0, t-w+1) .. t.
 *
 *   k_cache, v_cache [B, H, w, d] dtype, read and written in place
 *   q, k, v, y       [B, H, d]    dtype
 *   t >= 0;  d 64;  1 <= w <= 64
 *
 * Ordering: the bf16 kernel is launched as a programmatic dependent of the
 * previous work in `stream` and reads the ring slots other than t mod w and
 * (t-1) mod w before that work has finished. The kernel immediately before it
 * in the stream must therefore not write those slots of this cache; decode
 * steps on one cache issued in order (t after t-1, or t repeated) satisfy this.
 * The library records every ring that based_swa_prefill writes (the 256 most
 * recent), and the first decode on such a ring reads every slot only after
 * the previous work has finished, so prefill then decode back to back on one
 * stream is safe. A ring written by anything else (a copy, a caller's kernel)
 * needs another kernel, or a stream synchronisation, between that write and
 * the first decode.
 */
BASED_API based_status_t based_swa_decode(void* k_cache, void* v_cache, int64_t t,
                                const void* q, const void* k, const void* v, void* y,
                                int B, int H, int d, int w, float scale,
                                based_dtype_t dtype, cudaStream_t stream);

/*
 * based_baseconv_prefill -- the sequence-mixing core of a short gated
 * convolution (BaseConv) layer over N tokens. BASED §4 "The BASED Architecture"
 * (Additional mixers) and App. C "Extended Architecture Details" (Convolution):
 * a short convolution with a SiLU, combined with the projected input by an
 * elementwise product. The layer's input and output projections are per-token
 * affine maps that the caller applies; this call takes the two projected
 * streams u_gate and u_conv and computes, per sequence, channel and token t,
 *     c_t = bias + sum_{j=0}^{K-1} h[:, j] * u_conv[t - (K-1) + j]
 *           (causal and depthwise; u_conv is zero before token 0, so tap
 *            K-1 meets token t itself)
 *     y_t = u_gate[t] * SiLU(c_t),   SiLU(x) = x / (1 + exp(-x)).
 *
 *   u_gate, u_conv, y  [B, N, d] dtype, channels innermost; 16-byte aligned.
 *                      y must not overlap u_conv or state.
 *   h      [d, K] fp32 filter taps, 16-byte aligned, read only.
 *   bias   [d] fp32, 16-byte aligned, or NULL for none.
 *   state  [B, K-1, d] dtype, or NULL: written with u_conv of tokens
 *          N-K+1 .. N-1, oldest first, zeros for positions before token 0
 *          (the input of based_baseconv_decode). Unused when K = 1.
 *   B, N >= 1;  d a multiple of 4;  1 <= K <= 8 (else BASED_ERR_UNSUPPORTED).
 * Arithmetic in fp32; y rounded to the dtype. No workspace, no waits.
 */
BASED_API based_status_t based_baseconv_prefill(const void* u_gate, const void* u_conv, const float* h,
                                      const float* bias, void* y, void* state,
                                      int B, int N, int d, int K,
                                      based_dtype_t dtype, cudaStream_t stream);

/*
 * based_baseconv_decode -- one generated token per sequence through the same
 * filter: c = bias + sum_{j<K-1} h[:, j] * state[j] + h[:, K-1] * u_conv,
 * y = u_gate * SiLU(c); then the state drops its oldest row and appends u_conv.
 *
 *   state          [B, K-1, d] dtype, read and written in place (may be NULL when K = 1)
 *   u_gate, u_conv, y  [B, d] dtype
 *   h, bias, d, K  as for based_baseconv_prefill
 */
BASED_API based_status_t based_baseconv_decode(void* state, const void* u_gate, const void* u_conv,
                                     const float* h, const float* bias, void* y,
                                     int B, int d, int K, based_dtype_t dtype, cudaStream_t stream);

/*
 * based_get_last_error -- synchronises `stream`, then reports and clears the
 * device status word of the current device: BASED_ERR_TIMEOUT if a bounded
 * wait in a kernel expired since the last call, BASED_ERR_BOUNDS (debug
 * library only) if a kernel's store index check failed, BASED_ERR_CUDA if the
 * stream reported a CUDA error, else BASED_OK.
 */
BASED_API based_status_t based_get_last_error(cudaStream_t stream);

/* Static, NUL-terminated name of a status code ("BASED_OK", ...). */
BASED_API const char* based_status_string(based_status_t status);

/* Library version, major*10000 + minor*100 + patch. */
BASED_API int based_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BASED_H */

// Thin inline-PTX wrappers for the sm_100a tensor-core path: mbarriers with
// bounded waits, tcgen05 (TMEM allocation, MMA, commit, loads, fences) and the
// shared-memory matrix descriptors of the canonical no-swizzle layouts.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace based {
namespace tc {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete. Bounded: gives up after
// kWaitLimitNs (recording DEV_ERR_TIMEOUT in *status and raising *abort so the
// other roles stop waiting too), or as soon as another thread raised *abort.
// Returns false when it gave up.
//
// The poll loop is inline (a try_wait may suspend the thread until the phase
// completes, and wakes it within ~100 cycles); only the periodic check of the
// abort flag and the clock is out of line. A call to an out-of-line loop costs
// an instruction-cache miss in a large kernel on every wait that does not
// succeed at once, which measured several hundred cycles per hand-off.
// Periodic check of a wait that started at t0 (0: not yet timed): returns the
// start time, or 0 when the wait must give up.
static __device__ __noinline__ uint64_t mbar_wait_check(uint64_t t0, volatile int* abort, unsigned* status) {
    if (*abort) return 0;
    const uint64_t now = global_ns();
    if (t0 == 0) return now;
    if (now - t0 > kWaitLimitNs) {
        *abort = 1;
        atomicOr(status, DEV_ERR_TIMEOUT);
        return 0;
    }
    return t0;
}

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          unsigned* status) {
    uint64_t t0 = 0;
    for (uint32_t it = 1; !mbar_try_wait(bar, parity); ++it) {
        if ((it & 63u) == 0) {
            t0 = mbar_wait_check(t0, abort, status);
            if (t0 == 0) return false;
        }
    }
    return true;
}

// ------------------------------------------------------------------ fences

__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ------------------------------------------------------------------ TMEM

// Whole-warp calls. The allocated base address is written to *dst_smem.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// TMEM address of (lane, column).
__device__ __forceinline__ uint32_t tmem_addr(uint32_t base, uint32_t lane, uint32_t col) {
    return base + (lane << 16) + col;
}

// 32 lanes x 16 consecutive 32-bit columns: thread i of the warp gets lane (lane0 + i).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float* v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------ MMA

// Shared-memory matrix descriptor, canonical layout without swizzle: the
// operand is tiled into 8 x 16-byte core matrices stored as contiguous 128-byte
// blocks; `lbo` is the byte distance between core matrices adjacent along K,
// `sbo` the distance between core matrices adjacent along M (or N).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;           // descriptor version for sm_100
    return d;                                      // base offset 0, no swizzle
}

// Instruction descriptor of kind::f16 with bf16 A and B and an fp32 accumulator.
// a_mn / b_mn select MN-major (1) instead of K-major (0) operands.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn, bool b_mn) {
    return (1u << 4)                                   // D format: f32
           | (1u << 7)                                 // A format: bf16
           | (1u << 10)                                // B format: bf16
           | ((a_mn ? 1u : 0u) << 15) | ((b_mn ? 1u : 0u) << 16)
           | (static_cast<uint32_t>(N >> 3) << 17)
           | (static_cast<uint32_t>(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem], issued by one thread.
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on `bar` when every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

// ------------------------------------------------------------------ packing

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// a = 1 + s + s^2/2 for two scores at once with Blackwell's packed fp32 FMA
// (fma.rn.f32x2): the second-order Taylor weight of BASED's feature map.
__device__ __forceinline__ void taylor_pair(float s0, float s1, float& a0, float& a1) {
    asm("{\n\t.reg .b64 s, t, h, o;\n\t"
        "mov.b64 s, {%2, %3};\n\t"
        "mov.b64 h, 0x3F0000003F000000;\n\t"
        "mov.b64 o, 0x3F8000003F800000;\n\t"
        "fma.rn.f32x2 t, s, h, o;\n\t"
        "fma.rn.f32x2 s, s, t, o;\n\t"
        "mov.b64 {%0, %1}, s;\n\t}"
        : "=f"(a0), "=f"(a1)
        : "f"(s0), "f"(s1));
}

// (d0, d1) = (x - c)(1 + s) for two columns at once, as t = x - c, d = t s + t
// (sub.rn.f32x2 and fma.rn.f32x2): the score gradient of the Taylor weight.
__device__ __forceinline__ void dscore_pair(float x0, float x1, float c0, float c1, float s0, float s1, float& d0,
                                            float& d1) {
    asm("{\n\t.reg .b64 x, c, s, t;\n\t"
        "mov.b64 x, {%2, %3};\n\t"
        "mov.b64 c, {%4, %5};\n\t"
        "mov.b64 s, {%6, %7};\n\t"
        "sub.rn.f32x2 t, x, c;\n\t"
        "fma.rn.f32x2 t, t, s, t;\n\t"
        "mov.b64 {%0, %1}, t;\n\t}"
        : "=f"(d0), "=f"(d1)
        : "f"(x0), "f"(x1), "f"(c0), "f"(c1), "f"(s0), "f"(s1));
}

// (l0, l1) += (a0, a1) with the packed fp32 add.
__device__ __forceinline__ void add_pair(float& l0, float& l1, float a0, float a1) {
    asm("{\n\t.reg .b64 l, a;\n\t"
        "mov.b64 l, {%0, %1};\n\t"
        "mov.b64 a, {%2, %3};\n\t"
        "add.rn.f32x2 l, l, a;\n\t"
        "mov.b64 {%0, %1}, l;\n\t}"
        : "+f"(l0), "+f"(l1)
        : "f"(a0), "f"(a1));
}

__device__ __forceinline__ uint4 pack_bf16x8(const float* x) {
    return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                      pack_bf16x2(x[6], x[7]));
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t saddr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(saddr)
                 : "memory");
    return v;
}

__device__ __forceinline__ void st_shared_v4(uint32_t saddr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_shared_f32(uint32_t saddr, float v) {
    asm volatile("st.shared.f32 [%0], %1;" ::"r"(saddr), "f"(v) : "memory");
}

__device__ __forceinline__ float ld_shared_f32(uint32_t saddr) {
    float v;
    asm volatile("ld.shared.f32 %0, [%1];" : "=f"(v) : "r"(saddr) : "memory");
    return v;
}

}  // namespace tc
}  // namespace based

namespace based {
namespace tc {

// ------------------------------------------------------------------ 128-byte swizzled operands

// Descriptor of a tile stored as 8-row x 128-byte atoms (1024 B, 1024-aligned)
// with the 16-byte pieces of row r XOR-permuted by (r mod 8): the layout a TMA
// load with 128-byte swizzle produces. K-major operands step along K inside the
// 128-byte row by advancing `saddr`; `sbo` is the distance between 8-row atoms
// along M/N (K-major) or along K (MN-major); `lbo` is the distance between atoms
// along MN for MN-major operands wider than 64 bf16 (unused otherwise).
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;           // descriptor version for sm_100
    d |= static_cast<uint64_t>(2) << 61;           // 128-byte swizzle
    return d;
}

// The same for the 32-byte (layout 6) and 64-byte (layout 4) swizzles, whose
// atoms are 8 rows of 32 or 64 bytes: a K-major operand with rows of exactly
// that width (`sbo` = 8 rows) steps along K by advancing `saddr`.
__device__ __forceinline__ uint64_t smem_desc_swizzled(uint32_t saddr, uint32_t lbo, uint32_t sbo, int swizzle_bytes) {
    uint64_t d = 0;
    d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    const uint64_t mode = swizzle_bytes == 128 ? 2 : swizzle_bytes == 64 ? 4 : 6;
    d |= mode << 61;
    return d;
}

// Byte offset of 16-byte piece `chunk` (0..7) of row `row` inside a 128B-swizzled atom column.
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t chunk) {
    return row * 128u + ((chunk ^ (row & 7u)) << 4);
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// 1-D bulk copy global -> shared, completing `bar`'s transaction count. Both
// addresses 16-byte aligned, `bytes` a multiple of 16.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// 3-D tiled TMA load into shared memory, completing `bar`'s transaction count.
// Coordinates: x innermost (elements), then y, z; y may be negative or past the
// end (the box is zero-filled there); x must keep 16-byte alignment.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* tmap, uint64_t* bar, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
            dst),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

// Fetch a tensor map (a __grid_constant__ kernel parameter) into the TMA unit
// ahead of its first copy, which would otherwise wait for it.
__device__ __forceinline__ void prefetch_tensormap(const void* tmap) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tmap)) : "memory");
}

// Prefetch `bytes` (a multiple of 16) of global memory from `src` (16-byte
// aligned) into L2, with no completion to wait for.
__device__ __forceinline__ void prefetch_l2(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes)
                 : "memory");
}

// Prefetch the 3-D tile at (x, y, z) of a tensor map into L2 (no shared
// memory, no completion to wait for): later TMA loads of it hit L2.
__device__ __forceinline__ void tma_prefetch_3d(const void* tmap, int x, int y, int z) {
    asm volatile("cp.async.bulk.prefetch.tensor.3d.L2.global.tile [%0, {%1, %2, %3}];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(x), "r"(y), "r"(z)
                 : "memory");
}

}  // namespace tc
}  // namespace based

namespace based {
namespace tc {

// D[tmem] (+)= A[tmem] * B[smem]: the A operand (M rows = TMEM lanes, K packed
// two bf16 per 32-bit column, lower k in the low half) is read from tensor memory.
__device__ __forceinline__ void mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 16 consecutive 32-bit columns from registers: thread i writes lane (lane0 + i).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// 32 lanes x 8 consecutive 32-bit columns from registers.
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t* r) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

}  // namespace tc
}  // namespace based

namespace based {
namespace tc {

// ------------------------------------------------------------------ TMA stores

// 3-D tiled TMA store from shared memory (bulk-group completion). Rows past the
// tensor's extent are not written; the start coordinates must be >= 0 and x
// 16-byte aligned.
__device__ __forceinline__ void tma_store_3d(const void* tmap, uint32_t src, int x, int y, int z) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(tmap)),
        "r"(src), "r"(x), "r"(y), "r"(z)
        : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until every committed bulk store has finished reading its shared-memory source.
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }

// Wait until every committed bulk store has completed.
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

}  // namespace tc
}  // namespace based

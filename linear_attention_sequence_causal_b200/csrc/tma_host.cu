// Host-side TMA tensor-map encoding via cudaGetDriverEntryPoint (the library does not link libcuda).
#include <mutex>

#include "tma_host.h"

namespace based {
namespace {

using EncodeTiled = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                 const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiled encoder() {
    static EncodeTiled fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiled>(p);
    });
    return fn;
}

}  // namespace

bool make_tmap_bf16_3d_swizzle(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z,
                               uint32_t box_x, uint32_t box_y, int swizzle_bytes) {
    EncodeTiled fn = encoder();
    if (fn == nullptr) return false;
    CUtensorMapSwizzle sw;
    switch (swizzle_bytes) {
        case 32: sw = CU_TENSOR_MAP_SWIZZLE_32B; break;
        case 64: sw = CU_TENSOR_MAP_SWIZZLE_64B; break;
        case 128: sw = CU_TENSOR_MAP_SWIZZLE_128B; break;
        default: return false;
    }
    if (box_x * 2 > static_cast<uint32_t>(swizzle_bytes)) return false;
    const cuuint64_t dims[3] = {x, y, z};
    const cuuint64_t strides[2] = {x * 2, x * y * 2};          // bytes, dims 1 and 2
    const cuuint32_t box[3] = {box_x, box_y, 1};
    const cuuint32_t estride[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estride,
              CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tmap_bf16_3d(CUtensorMap* map, const void* base, uint64_t x, uint64_t y, uint64_t z, uint32_t box_x,
                       uint32_t box_y) {
    return make_tmap_bf16_3d_swizzle(map, base, x, y, z, box_x, box_y, 128);
}

}  // namespace based

// tmap.cu -- TMA tensor-map creation (host).  cuTensorMapEncodeTiled is a driver API
// call; it is resolved at run time through the runtime's entry-point query so that the
// library does not link libcuda and still loads on machines without a GPU driver.
#include "la_internal.cuh"
#include "tmap.cuh"

#include <mutex>

namespace la {
namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                             &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
        else
            (void)cudaGetLastError();
    });
    return fn;
}

}  // namespace

bool make_tmap_2d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, uint32_t elem_bytes,
                  uint64_t inner, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                  uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if ((reinterpret_cast<uintptr_t>(base) & 15u) || (row_stride_bytes & 15u)) return false;
    if (box_inner * elem_bytes > 128 && swizzle128) return false;
    const cuuint64_t dims[2] = {inner, rows};
    const cuuint64_t strides[1] = {row_stride_bytes};
    const cuuint32_t box[2] = {box_inner, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(map, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool make_tmap_3d(CUtensorMap *map, const void *base, CUtensorMapDataType dtype, uint32_t elem_bytes,
                  uint64_t inner, uint64_t rows, uint64_t outer, uint64_t row_pitch,
                  uint64_t outer_pitch, uint32_t box_inner, uint32_t box_rows, bool swizzle128) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    if ((reinterpret_cast<uintptr_t>(base) & 15u) || (row_pitch & 15u) || (outer_pitch & 15u))
        return false;
    if (box_inner * elem_bytes > 128 && swizzle128) return false;
    const cuuint64_t dims[3] = {inner, rows, outer};
    const cuuint64_t strides[2] = {row_pitch, outer_pitch};
    const cuuint32_t box[3] = {box_inner, box_rows, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(map, dtype, 3, const_cast<void *>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE,
                          swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace la

// tmap.cu -- TMA tensor-map encoding.  The driver's cuTensorMapEncodeTiled is
// fetched through the runtime (cudaGetDriverEntryPoint) so that the library
// does not link libcuda and can be loaded on a machine without a GPU driver.
#include <mutex>

#include "launch.h"

namespace moe {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn(cudaError_t* err) {
    static std::once_flag once;
    static EncodeTiledFn fn = nullptr;
    static cudaError_t status = cudaSuccess;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        status = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (status == cudaSuccess && q != cudaDriverEntryPointSuccess) status = cudaErrorNotSupported;
        fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    *err = status;
    return fn;
}

}  // namespace

cudaError_t make_tmap_u8_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_cols, uint32_t box_rows, int swizzle_bytes) {
    cudaError_t err;
    EncodeTiledFn fn = encode_fn(&err);
    if (!fn) return err == cudaSuccess ? cudaErrorNotSupported : err;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols};  // bytes between rows
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
                    estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                              uint32_t box_cols, uint32_t box_rows) {
    cudaError_t err;
    EncodeTiledFn fn = encode_fn(&err);
    if (!fn) return err == cudaSuccess ? cudaErrorNotSupported : err;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {cols * 2};  // bytes between rows
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t make_tmap_bf16_kchunks(CUtensorMap* map, const void* base, uint64_t rows, uint64_t cols,
                                   uint32_t box_rows, uint32_t box_chunks) {
    cudaError_t err;
    EncodeTiledFn fn = encode_fn(&err);
    if (!fn) return err == cudaSuccess ? cudaErrorNotSupported : err;
    // [rows, cols] viewed as (64 columns, rows, cols / 64 chunks): a box is
    // box_chunks consecutive 64-column chunks of box_rows rows, each chunk a
    // 128-byte-swizzled tile of its own in shared memory.
    const cuuint64_t dims[3] = {64, rows, cols / 64};
    const cuuint64_t strides[2] = {cols * 2, 128};  // bytes between rows, between chunks
    const cuuint32_t box[3] = {64, box_rows, box_chunks};
    const cuuint32_t estride[3] = {1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estride,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace moe

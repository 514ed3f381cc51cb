// Host-side TMA tensor-map encoding.  The CUDA driver entry point is looked up at run
// time through the CUDA runtime, so the library needs no link against libcuda.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

namespace fa {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// A 4-D bf16 tensor map whose box is 64 contiguous elements (128 bytes) by
// `box_rows` rows, loaded with the 128-byte swizzle.  dims are innermost first;
// stride_bytes[i] is the byte stride of dimension i + 1.  Out-of-range elements
// read as zero.  Returns false if the CUDA driver rejects the description.
inline bool make_tmap_bf16_4d(CUtensorMap* map, const void* base, const uint64_t dims[4],
                              const uint64_t stride_bytes[3], uint32_t box_rows)
{
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t gdim[4] = {dims[0], dims[1], dims[2], dims[3]};
    cuuint64_t gstride[3] = {stride_bytes[0], stride_bytes[1], stride_bytes[2]};
    cuuint32_t box[4] = {64, box_rows, 1, 1};
    cuuint32_t estride[4] = {1, 1, 1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// A 2-D fp32 tensor map over a row-major [rows, cols] matrix (cols contiguous,
// cols * 4 a multiple of 16) whose box is 32 columns (128 bytes) by 32 rows in
// the 128-byte swizzle: the layout of a warp's 32 rows staged in shared memory
// with 16-byte unit u of row r at position u ^ (r % 8).  Used as the target of TMA
// reductions.  Returns false if the CUDA driver rejects the description.
inline bool make_tmap_f32_2d_box32(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows)
{
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    cuuint64_t gdim[2] = {cols, rows};
    cuuint64_t gstride[1] = {cols * 4};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), gdim, gstride, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

} // namespace fa

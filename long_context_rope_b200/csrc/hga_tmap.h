// hga_tmap.h -- host-side creation of TMA tensor maps (cuTensorMapEncodeTiled,
// fetched through the runtime's driver entry-point query; no libcuda link).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

namespace hga {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

// Map over a row-major bf16 tensor [n_outer][n_rows][d] as (d, n_rows, n_outer):
// boxes of 64 elements (128 bytes) x box_rows rows x 1, 128-byte swizzle,
// zero fill outside the tensor. Returns false on failure.
inline bool make_rows_map(CUtensorMap* m, const void* base, int64_t n_outer, int64_t n_rows,
                          int d, int box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n_rows, (cuuint64_t)n_outer};
    cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n_rows * d * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over a row-major tensor of 1-byte elements (E4M3 codes) [n_outer][n_rows][d]
// as (d, n_rows, n_outer): boxes of 128 elements (128 bytes) x box_rows rows x
// 1, 128-byte swizzle, zero fill outside the tensor. Returns false on failure.
inline bool make_rows_map_u8(CUtensorMap* m, const void* base, int64_t n_outer, int64_t n_rows,
                             int d, int box_rows) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n_rows, (cuuint64_t)n_outer};
    cuuint64_t strides[2] = {(cuuint64_t)d, (cuuint64_t)n_rows * d};
    cuuint32_t box[3] = {128, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Map over queries [B][n_tok][Hq][d] bf16 as (d, Hq, n_tok, B): boxes of
// 64 elements x box_heads heads x box_tok tokens x 1, 128-byte swizzle.
inline bool make_query_map(CUtensorMap* m, const void* base, int64_t B, int64_t n_tok, int Hq,
                           int d, int box_heads, int box_tok) {
    EncodeTiledFn fn = encode_tiled_fn();
    if (fn == nullptr) return false;
    cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)Hq, (cuuint64_t)n_tok, (cuuint64_t)B};
    cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)Hq * d * 2,
                             (cuuint64_t)n_tok * Hq * d * 2};
    cuuint32_t box[4] = {64, (cuuint32_t)box_heads, (cuuint32_t)box_tok, 1};
    cuuint32_t es[4] = {1, 1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
              es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace hga

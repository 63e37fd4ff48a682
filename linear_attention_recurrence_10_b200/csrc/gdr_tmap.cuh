// gdr_tmap.cuh -- host-side tensor maps for the TMA tensor copies of the
// attention decode and the prefill's prep kernel.
#pragma once

#include <cuda.h>  // CUtensorMap and its encoder's types (fetched from the driver at run time)
#include <cuda_runtime.h>

#include <cstdint>

namespace gdr {

using EncodeTiledFn = decltype(&cuTensorMapEncodeTiled);

// The driver's tensor-map encoder, looked up once through the runtime (no
// link-time dependency on the driver library); null if the driver lacks it.
inline EncodeTiledFn encode_tiled() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *f = nullptr;
        cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &f, 12000, cudaEnableDefault,
                                             &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            (void)cudaGetLastError();
            return nullptr;
        }
        return reinterpret_cast<EncodeTiledFn>(f);
    }();
    return fn;
}

// A row-major bf16 matrix of `rows` rows, `cols` elements used per row and
// `row_bytes` between rows, copied in boxes of box_cols x box_rows with the
// 128-byte swizzle (box_cols * 2 must be 128); elements outside the matrix
// read as zero.  False when the encoder is missing or refuses the shape: the
// base must be 16-byte aligned and row_bytes a multiple of 16.
inline bool encode_bf16_2d(CUtensorMap *m, const void *base, uint64_t cols, uint64_t rows,
                           uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows) {
    const EncodeTiledFn fn = encode_tiled();
    if (!fn || (reinterpret_cast<uintptr_t>(base) & 15u) || (row_bytes & 15u) || rows == 0 ||
        cols * 2 > row_bytes)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t elem_strides[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box,
              elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace gdr

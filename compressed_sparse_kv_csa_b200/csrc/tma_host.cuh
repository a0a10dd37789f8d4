// tma_host.cuh -- host-side tensor-map encoding for the TMA loads (no libcuda link: the driver
// entry point is looked up through the runtime).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

namespace csa {
namespace tma {

inline PFN_cuTensorMapEncodeTiled_v12000 encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

// Row-major bf16 matrix [rows, cols] (row stride cols*2 bytes) read in boxes of 64 columns x
// box_rows rows with the 128-byte swizzle; rows outside the matrix read as zeros.
inline bool encode_bf16_rows(CUtensorMap *m, const void *base, uint64_t rows, uint64_t cols, uint32_t box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
    if (!enc || rows == 0 || cols % 64 || box_rows == 0 || box_rows > 256) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Rows of `row_bytes` bytes (row stride row_bytes) read as bytes in boxes of the whole row x
// box_rows rows, with the 64-byte swizzle (row_bytes must be 64); rows outside read as zeros.
// Used for packed FP4 operands (two E2M1 codes per byte, 64 bytes = 128 elements per row).
inline bool encode_u8_rows_sw64(CUtensorMap *m, const void *base, uint64_t rows, uint32_t row_bytes,
                                uint32_t box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
    if (!enc || rows == 0 || row_bytes != 64 || box_rows == 0 || box_rows > 256) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    const cuuint32_t box[2] = {row_bytes, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Every 4th row of a [rows, 64]-byte matrix: the 3-D view {64 bytes, 4 (row mod 4), rows / 4} read
// in boxes of 64 bytes x 1 x box_rows with the 64-byte swizzle, so that box (0, j, y) holds rows
// 4y + j, 4(y+1) + j, ...; rows must be a multiple of 4; rows outside read as zeros.
inline bool encode_u8_rows_sw64_stride4(CUtensorMap *m, const void *base, uint64_t rows, uint32_t box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
    if (!enc || rows < 4 || rows % 4 || box_rows == 0 || box_rows > 256) return false;
    const cuuint64_t dims[3] = {64, 4, (cuuint64_t)(rows / 4)};
    const cuuint64_t strides[2] = {64, 256};
    const cuuint32_t box[3] = {64, 1, box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A vector of 32-bit words viewed as rows of 4 words ({4, words / 4}), read in boxes of 4 x
// box_rows without swizzle; words must be a multiple of 4; rows outside read as zeros.
inline bool encode_u32_quads(CUtensorMap *m, const void *base, uint64_t words, uint32_t box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = encoder();
    if (!enc || words < 4 || words % 4 || box_rows == 0 || box_rows > 256) return false;
    const cuuint64_t dims[2] = {4, (cuuint64_t)(words / 4)};
    const cuuint64_t strides[1] = {16};
    const cuuint32_t box[2] = {4, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

} // namespace tma
} // namespace csa

// tmap.h -- host-side encoding of the 2-D tensor maps the row kernels copy
// with (rows of BF16 viewed as 128-byte lines, SWIZZLE_128B).
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

namespace mb {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// A BF16 buffer of `lines` 128-byte lines (64 elements each), copied in boxes
// of `box_lines` lines.  Returns false when the driver rejects the map.
inline bool encode_line_map(CUtensorMap* map, const void* base, uint64_t lines, uint32_t box_lines) {
    std::memset(map, 0, sizeof(*map));
    auto fn = tensor_map_encoder();
    if (fn == nullptr || lines == 0 || box_lines == 0 || box_lines > 256) return false;
    cuuint64_t dims[2] = {64, lines};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, box_lines};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
                    estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// A row-major 2-D array of `rows` x `cols` elements of `elem_bytes` bytes
// (row pitch `pitch_bytes`), copied in boxes of box_rows x box_cols (with
// `swizzle` in shared memory); rows and columns past the end read as zero.
inline bool encode_2d_map(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t elem_bytes, const void* base,
                          uint64_t rows, uint64_t cols, uint64_t pitch_bytes, uint32_t box_rows, uint32_t box_cols,
                          CUtensorMapSwizzle swizzle = CU_TENSOR_MAP_SWIZZLE_NONE) {
    std::memset(map, 0, sizeof(*map));
    auto fn = tensor_map_encoder();
    if (fn == nullptr || rows == 0 || cols == 0 || box_rows == 0 || box_rows > 256 || box_cols == 0 ||
        box_cols * elem_bytes % 16 != 0)
        return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {pitch_bytes};
    cuuint32_t box[2] = {box_cols, box_rows};
    cuuint32_t estride[2] = {1, 1};
    CUresult r = fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                    swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace mb

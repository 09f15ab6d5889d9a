// Host-side construction of TMA tensor maps (driver entry point fetched
// through the runtime, so the library links only against cudart).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "internal.h"

namespace dsa {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult qres;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &qres) == cudaSuccess &&
            qres == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

}  // namespace

namespace {

bool make_map_sw128(CUtensorMap *map, CUtensorMapDataType type, uint32_t box_cols, const void *base, uint64_t rows,
                    uint64_t cols, uint64_t pitch_bytes, uint32_t box_rows) {
    auto encode = get_encode_fn();
    if (!encode) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, type, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace

bool make_map_bf16_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                         uint32_t box_rows) {
    return make_map_sw128(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 64, base, rows, cols, pitch_bytes, box_rows);
}

bool make_map_u8_sw128(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                       uint32_t box_rows) {
    return make_map_sw128(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 128, base, rows, cols, pitch_bytes, box_rows);
}

bool make_map_f32(CUtensorMap *map, const void *base, uint64_t rows, uint64_t cols, uint64_t pitch_bytes,
                  uint32_t box_rows, uint32_t box_cols) {
    auto encode = get_encode_fn();
    if (!encode) return false;
    const cuuint64_t dims[2] = {cols, rows};
    const cuuint64_t strides[1] = {pitch_bytes};
    const cuuint32_t box[2] = {box_cols, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

}  // namespace dsa

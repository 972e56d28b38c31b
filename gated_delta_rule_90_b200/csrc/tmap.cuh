// Host-side construction of 2-D TMA tensor maps (driver entry point fetched
// through the runtime, so the library links only the static CUDA runtime).
#pragma once
#include <cuda.h>
#include <cudaTypedefs.h>

namespace gdr_host {
namespace tmap {

inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = (PFN_cuTensorMapEncodeTiled_v12000)p;
    }
    return fn;
}

// 2-D tensor map: inner extent `inner` elements, `rows` rows, row pitch
// `pitch` bytes, box box0 x box1, zero fill out of bounds.
inline bool make_map(CUtensorMap *m, CUtensorMapDataType type, const void *base, uint64_t inner,
                     uint64_t rows, uint64_t pitch, uint32_t box0, uint32_t box1,
                     CUtensorMapSwizzle swz) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, rows};
    cuuint64_t strides[1] = {pitch};
    cuuint32_t box[2] = {box0, box1};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, type, 2, const_cast<void *>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

constexpr CUtensorMapDataType kBF = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
constexpr CUtensorMapDataType kF32 = CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
constexpr CUtensorMapSwizzle kSW = CU_TENSOR_MAP_SWIZZLE_128B;
constexpr CUtensorMapSwizzle kNoSW = CU_TENSOR_MAP_SWIZZLE_NONE;

}  // namespace tmap
}  // namespace gdr_host

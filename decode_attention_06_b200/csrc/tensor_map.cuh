// tensor_map.cuh -- host-side construction of TMA tensor maps for bf16
// tensors.  The driver's cuTensorMapEncodeTiled is reached through the
// runtime's entry-point query, so the library does not link libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <stdint.h>

namespace gqla {

inline PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// Tiled map of `rank` (2 or 3) dimensions: dims[0] is the contiguous one,
// strides_bytes[i] is the byte stride of dims[i + 1].  Out-of-range elements
// of a box read as zero; a store drops them.
inline bool make_map(CUtensorMap *map, CUtensorMapDataType dtype, const void *base, int rank,
                     const uint64_t *dims, const uint64_t *strides_bytes, const uint32_t *box,
                     CUtensorMapSwizzle swizzle) {
    auto fn = tensor_map_encoder();
    if (!fn || rank < 2 || rank > 3) return false;
    cuuint64_t d[3], s[2];
    cuuint32_t b[3], e[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        b[i] = box[i];
    }
    for (int i = 0; i + 1 < rank; ++i) s[i] = strides_bytes[i];
    return fn(map, dtype, rank, const_cast<void *>(base), d, s, b, e,
              CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline bool make_bf16_map(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                          const uint64_t *strides_bytes, const uint32_t *box,
                          CUtensorMapSwizzle swizzle) {
    return make_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides_bytes, box,
                    swizzle);
}

}  // namespace gqla

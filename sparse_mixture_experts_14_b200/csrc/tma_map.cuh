// Host-side TMA tensor maps for bf16 operands (128-byte swizzle, zero fill out
// of bounds).  The encoder is the driver's cuTensorMapEncodeTiled, fetched once
// through the runtime so the library needs no link-time libcuda.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace moe {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The encoder, resolved on first use (thread-safe static initialisation); null if unavailable.
inline EncodeTiledFn tensor_map_encoder() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess) {
            cudaGetLastError();
            return nullptr;
        }
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// bf16 tensor map; dims/strides innermost first, strides in bytes, box in elements.
inline bool encode_bf16_map(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims,
                            const cuuint64_t* strides, const cuuint32_t* box) {
    const EncodeTiledFn fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// rows x K matrix, K contiguous: box K_box x box_rows
inline bool map_matrix(CUtensorMap* m, const void* base, size_t rows, int K, int k_box, int box_rows) {
    cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    cuuint32_t box[2] = {(cuuint32_t)k_box, (cuuint32_t)box_rows};
    return encode_bf16_map(m, base, 2, dims, strides, box);
}

// E x R x K weights, K contiguous: box K_box x box_rows x 1
inline bool map_expert_weights(CUtensorMap* m, const void* base, int E, int R, int K, int k_box, int box_rows) {
    cuuint64_t dims[3] = {(cuuint64_t)K, (cuuint64_t)R, (cuuint64_t)E};
    cuuint64_t strides[2] = {(cuuint64_t)K * 2, (cuuint64_t)R * K * 2};
    cuuint32_t box[3] = {(cuuint32_t)k_box, (cuuint32_t)box_rows, 1};
    return encode_bf16_map(m, base, 3, dims, strides, box);
}

}  // namespace moe

// tmap.h -- host-side TMA tensor maps for the (rows x 128 columns) bf16 slabs of one
// head (q, k, v, o are (B, H, T, 128) contiguous): a 3-D view (128 columns, T rows,
// heads) with a (64 columns x box_rows rows) box and the 128-byte swizzle, so that
// rows outside [0, T) of a head read as zero and a store clips them.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace falcon {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                  CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                  CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled from the driver, resolved once per process: a function-local
// static is initialised exactly once even when several host threads make their first
// call together. nullptr when the driver does not provide it.
inline EncodeTiledFn encode_tiled_fn() {
    static const EncodeTiledFn fn = []() -> EncodeTiledFn {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(ptr);
        return nullptr;
    }();
    return fn;
}

// (128 columns, T rows, heads) bf16 view with (64 x box_rows) boxes, 128-byte swizzle.
inline bool map_head_rows(CUtensorMap *m, const void *base, int T, long long heads, int box_rows) {
    const EncodeTiledFn fn = encode_tiled_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {128, (cuuint64_t)T, (cuuint64_t)heads};
    cuuint64_t strides[2] = {128 * 2, (cuuint64_t)T * 128 * 2};
    cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
    cuuint32_t es[3] = {1, 1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base), dims, strides, box, es,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace falcon

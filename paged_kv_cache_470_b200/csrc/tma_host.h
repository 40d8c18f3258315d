// Host side of the TMA tile loads: the tensor map of one cache tensor.
#pragma once

#include "pagedkv.h"

#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

namespace pkv_host {

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// View one cache tensor [num_blocks][16][Hkv][D] as a 4-D map whose dimensions
// are (column, row, kv head, block) -- rows inside heads, so each head's 16
// rows land as one contiguous 128B-swizzled 2 KB tile -- with a box of
// 64 columns x 16 rows x HG heads x 1 block.
inline bool make_cache_map(CUtensorMap *tm, const void *cache, int num_blocks, int Hkv, int D, int hg, int dtype)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc)
        return false;
    const cuuint64_t dims[4] = {static_cast<cuuint64_t>(D), 16, static_cast<cuuint64_t>(Hkv),
                                static_cast<cuuint64_t>(num_blocks)};
    const cuuint64_t strides[3] = {static_cast<cuuint64_t>(Hkv) * D * 2, static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(16) * Hkv * D * 2};
    const cuuint32_t box[4] = {64, 16, static_cast<cuuint32_t>(hg), 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt =
        dtype == KV_DTYPE_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return enc(tm, dt, 4, const_cast<void *>(cache), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A stack of `layers` such caches, layer l starting layer_stride_bytes * l
// after the first, as a 5-D map (column, row, kv head, block, layer) with the
// same box and one layer per box.
inline bool make_layered_cache_map(CUtensorMap *tm, const void *cache, int num_blocks, int Hkv, int D, int hg,
                                   int dtype, int layers, unsigned long long layer_stride_bytes)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc || layers < 1)
        return false;
    const cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), 16, static_cast<cuuint64_t>(Hkv),
                                static_cast<cuuint64_t>(num_blocks), static_cast<cuuint64_t>(layers)};
    const cuuint64_t strides[4] = {static_cast<cuuint64_t>(Hkv) * D * 2, static_cast<cuuint64_t>(D) * 2,
                                   static_cast<cuuint64_t>(16) * Hkv * D * 2,
                                   static_cast<cuuint64_t>(layer_stride_bytes)};
    const cuuint32_t box[5] = {64, 16, static_cast<cuuint32_t>(hg), 1, 1};
    const cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    const CUtensorMapDataType dt =
        dtype == KV_DTYPE_FP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return enc(tm, dt, 5, const_cast<void *>(cache), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pkv_host

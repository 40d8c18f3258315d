// kv_cache_append: scatter each new token's K and V rows into its block slot.
//
// "Module 23: Serving", section 23.4 (Paged Attention): blocks of 16 tokens are
// filled as a sequence grows; a slot is block * 16 + offset within the block.
//
// Layout: the row of token i in k_new/v_new is Hkv * D contiguous bf16; the
// destination row in the cache is cache[slot / 16][slot % 16][:][:], also
// Hkv * D contiguous bf16. One thread moves one 16-byte chunk of one row with a
// 128-bit load and store, so a warp covers 512 contiguous bytes.
#include "pkv_device.cuh"
#include "nvtx_range.h"
#include "pagedkv.h"

#include <cuda_runtime.h>

namespace pkv {

__global__ void __launch_bounds__(256) append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                                                     uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                                     const int64_t *__restrict__ slot_mapping, int T,
                                                     int64_t slot_limit, int chunks_per_row, int32_t *error_flag)
{
    // The cache may still be read by the previous kernel in the stream.
    grid_dependency_wait();
    grid_launch_dependents();
    const int64_t per_tensor = static_cast<int64_t>(T) * chunks_per_row;
    const int64_t total = 2 * per_tensor;
    for (int64_t idx = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const bool is_v = idx >= per_tensor;
        const int64_t rem = is_v ? idx - per_tensor : idx;
        const int64_t i = rem / chunks_per_row;
        const int64_t ch = rem - i * chunks_per_row;
        const int64_t slot = __ldg(slot_mapping + i);
        if (slot < 0)
            continue;
        if (slot >= slot_limit) {
            if (error_flag && ch == 0 && !is_v)
                atomicOr(error_flag, KV_STATUS_BAD_SLOT);
            continue;
        }
        const uint4 *src = (is_v ? v_new : k_new) + i * chunks_per_row + ch;
        uint4 *dst = (is_v ? v_cache : k_cache) + slot * chunks_per_row + ch;
        *dst = __ldg(src);
    }
}

}  // namespace pkv

extern "C" kv_status kv_cache_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                                     const int64_t *slot_mapping, int T, int num_blocks, int Hkv, int D, int dtype,
                                     int32_t *error_flag, kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("kv_cache_append");
    if (T < 0 || num_blocks < 1 || Hkv < 1 || (dtype != KV_DTYPE_BF16 && dtype != KV_DTYPE_FP16) || (D != 64 && D != 128))
        return KV_ERR_ARG;
    if (T == 0)
        return KV_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping)
        return KV_ERR_ARG;
    auto misaligned = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
    if (misaligned(k_new) || misaligned(v_new) || misaligned(k_cache) || misaligned(v_cache) ||
        (reinterpret_cast<uintptr_t>(slot_mapping) & 7u))
        return KV_ERR_ARG;
    const int chunks_per_row = Hkv * D * 2 / 16;
    const int64_t total = 2ll * T * chunks_per_row;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 65535)
        blocks = 65535;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = 0;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t err = cudaLaunchKernelEx(&cfg, pkv::append_kernel, static_cast<const uint4 *>(k_new),
                                         static_cast<const uint4 *>(v_new), static_cast<uint4 *>(k_cache),
                                         static_cast<uint4 *>(v_cache), slot_mapping, T,
                                         static_cast<int64_t>(num_blocks) * pkv::kBlockTokens, chunks_per_row,
                                         error_flag);
    return err == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

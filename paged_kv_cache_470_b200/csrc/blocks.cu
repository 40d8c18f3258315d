// Whole-block moves over a list of cache tensors (each [num_blocks][16][Hkv][D],
// any 2-byte element type: the kernels move bytes), typically every layer's K and
// V cache in one launch:
//
//   kv_cache_copy_blocks    cache[dst[i]] = cache[src[i]]     copy-on-write of a
//                           shared, partly filled block ("Designing an LLM serving
//                           system", section "Paged attention": when sequences
//                           diverge, the shared block is copied on write)
//   kv_cache_gather_blocks  out[i] = cache[ids[i]]            swap-out: pack a
//                           preempted sequence's blocks for one host copy
//   kv_cache_scatter_blocks cache[ids[i]] = in[i]             swap-in ("Designing an
//                           LLM serving system", section "Scheduling: when prefill
//                           meets decode": a preempted sequence's blocks are
//                           swapped out and back)
//
// One warp moves one block of one tensor with 16-byte loads and stores (16 * Hkv
// * D * 2 bytes, a multiple of 256): each lane issues four loads before their four
// stores, and a grid of resident CTAs strides over the (tensor, block) items.
#include "pkv_device.cuh"
#include "nvtx_range.h"
#include "pagedkv.h"

#include <cuda_runtime.h>

#include <atomic>

namespace pkv {

constexpr int kMaxMoveCaches = 128;

struct CacheList {
    uint4 *p[kMaxMoveCaches];
};

// Work item w = cache index (w / n) and pair (w % n), one warp each.
// mode 0: cache[dst_ids[i]] = cache[src_ids[i]]; mode 1: buf[c][i] = cache_c[src_ids[i]];
// mode 2: cache_c[dst_ids[i]] = buf[c][i]. Ids outside [0, num_blocks) are skipped and
// flagged. In mode 0 no block may be both a source and a destination of one call, and
// destinations are distinct; in mode 2 destinations are distinct.
__global__ void __launch_bounds__(256) block_move_kernel(const __grid_constant__ CacheList caches, int n_caches,
                                                         uint4 *buf, const int32_t *__restrict__ src_ids,
                                                         const int32_t *__restrict__ dst_ids, int n, int num_blocks,
                                                         int chunks_per_block, int mode, int32_t *error_flag)
{
    grid_dependency_wait();
    grid_launch_dependents();
    const int lane = threadIdx.x & 31;
    const long long warps = (static_cast<long long>(gridDim.x) * blockDim.x) >> 5;
    const long long total = static_cast<long long>(n) * n_caches;
    for (long long w = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5; w < total; w += warps) {
        const int c = static_cast<int>(w / n);
        const int i = static_cast<int>(w - static_cast<long long>(c) * n);
        const long long s = (mode != 2) ? __ldg(src_ids + i) : 0;
        const long long d = (mode != 1) ? __ldg(dst_ids + i) : 0;
        if ((mode != 2 && (s < 0 || s >= num_blocks)) || (mode != 1 && (d < 0 || d >= num_blocks))) {
            if (error_flag && lane == 0)
                atomicOr(error_flag, KV_STATUS_BAD_BLOCK_ID);
            continue;
        }
        uint4 *cache = caches.p[c];
        uint4 *packed = buf + (static_cast<long long>(c) * n + i) * chunks_per_block;
        const uint4 *src = (mode == 2) ? packed : cache + s * chunks_per_block;
        uint4 *dst = (mode == 1) ? packed : cache + d * chunks_per_block;
        int k = lane;
        for (; k + 96 < chunks_per_block; k += 128) {
            const uint4 a0 = src[k], a1 = src[k + 32], a2 = src[k + 64], a3 = src[k + 96];
            dst[k] = a0;
            dst[k + 32] = a1;
            dst[k + 64] = a2;
            dst[k + 96] = a3;
        }
        for (; k < chunks_per_block; k += 32)
            dst[k] = src[k];
    }
}

}  // namespace pkv

namespace {

// CTAs of block_move_kernel (256 threads) resident on the current device at once, per device.
long long resident_move_ctas()
{
    constexpr int kMaxDevices = 64;
    static std::atomic<long long> cache[kMaxDevices];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return 0;
    long long v = cache[dev].load();
    if (v == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pkv::block_move_kernel, 256, 0) != cudaSuccess ||
            sms < 1 || per_sm < 1)
            return 0;
        v = static_cast<long long>(sms) * per_sm;
        cache[dev].store(v);
    }
    return v;
}

kv_status launch_move(void *const *caches, int n_caches, void *buf, const int32_t *src_ids, const int32_t *dst_ids,
                      int n, int num_blocks, int Hkv, int D, int dtype, int mode, int32_t *error_flag,
                      kv_stream_t stream)
{
    if (n < 0 || n_caches < 0 || n_caches > pkv::kMaxMoveCaches || num_blocks < 1 || Hkv < 1 || D < 8 ||
        D % 8 != 0 || (dtype != KV_DTYPE_BF16 && dtype != KV_DTYPE_FP16))
        return KV_ERR_ARG;
    if (n == 0 || n_caches == 0)
        return KV_OK;
    if (!caches || (mode != 0 && !buf) || (mode != 2 && !src_ids) || (mode != 1 && !dst_ids))
        return KV_ERR_ARG;
    if (reinterpret_cast<uintptr_t>(buf) & 15u)
        return KV_ERR_ARG;
    pkv::CacheList list = {};
    for (int c = 0; c < n_caches; ++c) {
        if (!caches[c] || (reinterpret_cast<uintptr_t>(caches[c]) & 15u))
            return KV_ERR_ARG;
        list.p[c] = static_cast<uint4 *>(caches[c]);
    }
    const int chunks = 16 * Hkv * D * 2 / 16;
    const int threads = 256;
    long long blocks = (static_cast<long long>(n) * n_caches * 32 + threads - 1) / threads;
    const long long resident = resident_move_ctas();  // one wave: the rest is strided over
    if (resident <= 0)
        return KV_ERR_CUDA;
    if (blocks > resident)
        blocks = resident;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(threads);
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, pkv::block_move_kernel, list, n_caches, static_cast<uint4 *>(buf),
                                             src_ids, dst_ids, n, num_blocks, chunks, mode, error_flag);
    return e == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

}  // namespace

extern "C" kv_status kv_cache_copy_blocks(void *const *caches, int n_caches, const int32_t *src_ids,
                                          const int32_t *dst_ids, int n, int num_blocks, int Hkv, int D, int dtype,
                                          int32_t *error_flag, kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("kv_cache_copy_blocks");
    return launch_move(caches, n_caches, nullptr, src_ids, dst_ids, n, num_blocks, Hkv, D, dtype, 0, error_flag,
                       stream);
}

extern "C" kv_status kv_cache_gather_blocks(void *out, void *const *caches, int n_caches, const int32_t *block_ids,
                                            int n, int num_blocks, int Hkv, int D, int dtype, int32_t *error_flag,
                                            kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("kv_cache_gather_blocks");
    return launch_move(caches, n_caches, out, block_ids, nullptr, n, num_blocks, Hkv, D, dtype, 1, error_flag,
                       stream);
}

extern "C" kv_status kv_cache_scatter_blocks(void *const *caches, int n_caches, const void *in,
                                             const int32_t *block_ids, int n, int num_blocks, int Hkv, int D,
                                             int dtype, int32_t *error_flag, kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("kv_cache_scatter_blocks");
    return launch_move(caches, n_caches, const_cast<void *>(in), nullptr, block_ids, n, num_blocks, Hkv, D, dtype, 2,
                       error_flag, stream);
}

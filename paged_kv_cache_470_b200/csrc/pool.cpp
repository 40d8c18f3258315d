// Host block pool: free list and reference counts for the paged KV cache.
//
// "Module 23: Serving", section 23.4 (Paged Attention): fixed-size blocks are
// handed out as a sequence grows, and sequences sharing a prefix can share its
// blocks. "Designing an LLM serving system", section "Paged attention": a page
// table per sequence maps logical positions to physical blocks; shared blocks
// for a common prompt. "Module 23: Serving", Exercise (extend): unused space is
// at most one partly filled block per request.
//
// The pool owns no device memory: it only decides which physical block ids
// are in use. Free ids sit on a stack (most recently freed first), reference
// counts in a flat array. Every call validates its whole request before
// changing anything, so a failed call leaves the pool as it was.
#include "nvtx_range.h"
#include "pagedkv.h"

#include <mutex>
#include <new>
#include <unordered_map>
#include <vector>

namespace {

struct BlockPool {
    std::mutex mu;
    std::vector<int32_t> free_ids;  // stack; back() is handed out next
    std::vector<int32_t> refcount;  // per block; 0 = free
};

BlockPool *as_pool(void *p) { return static_cast<BlockPool *>(p); }
const BlockPool *as_pool(const void *p) { return static_cast<const BlockPool *>(p); }

}  // namespace

extern "C" kv_status kv_pool_create(int num_blocks, void **pool_out)
{
    if (num_blocks < 0 || !pool_out)
        return KV_ERR_ARG;
    BlockPool *p = new (std::nothrow) BlockPool;
    if (!p)
        return KV_ERR_OOM;
    try {
        p->refcount.assign(static_cast<size_t>(num_blocks), 0);
        p->free_ids.resize(static_cast<size_t>(num_blocks));
        for (int i = 0; i < num_blocks; ++i)
            p->free_ids[static_cast<size_t>(i)] = num_blocks - 1 - i;  // block 0 comes out first
    } catch (...) {
        delete p;
        return KV_ERR_OOM;
    }
    *pool_out = p;
    return KV_OK;
}

extern "C" void kv_pool_destroy(void *pool) { delete as_pool(pool); }

extern "C" kv_status kv_pool_alloc(void *pool, int n, int32_t *ids_out)
{
    if (!pool || n < 0 || (n > 0 && !ids_out))
        return KV_ERR_ARG;
    BlockPool *p = as_pool(pool);
    std::lock_guard<std::mutex> lock(p->mu);
    if (static_cast<size_t>(n) > p->free_ids.size())
        return KV_ERR_OOM;
    for (int i = 0; i < n; ++i) {
        const int32_t id = p->free_ids.back();
        p->free_ids.pop_back();
        p->refcount[static_cast<size_t>(id)] = 1;
        ids_out[i] = id;
    }
    return KV_OK;
}

extern "C" kv_status kv_pool_incref(void *pool, const int32_t *ids, int n)
{
    if (!pool || n < 0 || (n > 0 && !ids))
        return KV_ERR_ARG;
    BlockPool *p = as_pool(pool);
    std::lock_guard<std::mutex> lock(p->mu);
    const int64_t nb = static_cast<int64_t>(p->refcount.size());
    for (int i = 0; i < n; ++i)
        if (ids[i] < 0 || ids[i] >= nb || p->refcount[static_cast<size_t>(ids[i])] <= 0)
            return KV_ERR_STATE;
    for (int i = 0; i < n; ++i)
        ++p->refcount[static_cast<size_t>(ids[i])];
    return KV_OK;
}

extern "C" kv_status kv_pool_free(void *pool, const int32_t *ids, int n)
{
    if (!pool || n < 0 || (n > 0 && !ids))
        return KV_ERR_ARG;
    BlockPool *p = as_pool(pool);
    std::lock_guard<std::mutex> lock(p->mu);
    const int64_t nb = static_cast<int64_t>(p->refcount.size());
    // an id may appear several times in one call: count drops per id first
    std::unordered_map<int32_t, int> drops;
    for (int i = 0; i < n; ++i) {
        if (ids[i] < 0 || ids[i] >= nb)
            return KV_ERR_STATE;
        if (++drops[ids[i]] > p->refcount[static_cast<size_t>(ids[i])])
            return KV_ERR_STATE;
    }
    for (int i = 0; i < n; ++i) {
        int32_t &rc = p->refcount[static_cast<size_t>(ids[i])];
        if (--rc == 0)
            p->free_ids.push_back(ids[i]);
    }
    return KV_OK;
}

extern "C" int kv_pool_num_free(const void *pool)
{
    if (!pool)
        return -1;
    BlockPool *p = const_cast<BlockPool *>(as_pool(pool));
    std::lock_guard<std::mutex> lock(p->mu);
    return static_cast<int>(p->free_ids.size());
}

extern "C" int kv_pool_num_blocks(const void *pool)
{
    if (!pool)
        return -1;
    return static_cast<int>(as_pool(pool)->refcount.size());
}

extern "C" int kv_pool_refcount(const void *pool, int32_t id)
{
    if (!pool)
        return -1;
    BlockPool *p = const_cast<BlockPool *>(as_pool(pool));
    std::lock_guard<std::mutex> lock(p->mu);
    if (id < 0 || static_cast<size_t>(id) >= p->refcount.size())
        return -1;
    return p->refcount[static_cast<size_t>(id)];
}

extern "C" kv_status kv_pool_append_slots(void *pool, int32_t *block_tables, int W, int32_t *context_lens, int B,
                                          int64_t *slot_mapping_out)
{
    pkv_host::NvtxRange nvtx_range("kv_pool_append_slots");
    if (!pool || B < 0 || W < 1 || (B > 0 && (!block_tables || !context_lens || !slot_mapping_out)))
        return KV_ERR_ARG;
    BlockPool *p = as_pool(pool);
    std::lock_guard<std::mutex> lock(p->mu);
    const int64_t nb = static_cast<int64_t>(p->refcount.size());
    // validate the whole step first
    size_t need = 0;
    for (int b = 0; b < B; ++b) {
        const int c = context_lens[b];
        if (c < 0 || c / KV_BLOCK_TOKENS >= W)
            return KV_ERR_ARG;
        if (c % KV_BLOCK_TOKENS == 0) {
            ++need;
        } else {
            const int32_t tail = block_tables[static_cast<size_t>(b) * W + c / KV_BLOCK_TOKENS];
            if (tail < 0 || tail >= nb || p->refcount[static_cast<size_t>(tail)] <= 0)
                return KV_ERR_STATE;
            if (p->refcount[static_cast<size_t>(tail)] > 1)
                return KV_ERR_STATE;  // would write into a block another sequence reads
        }
    }
    if (need > p->free_ids.size())
        return KV_ERR_OOM;
    for (int b = 0; b < B; ++b) {
        const int c = context_lens[b];
        int32_t *row = block_tables + static_cast<size_t>(b) * W;
        if (c % KV_BLOCK_TOKENS == 0) {
            const int32_t id = p->free_ids.back();
            p->free_ids.pop_back();
            p->refcount[static_cast<size_t>(id)] = 1;
            row[c / KV_BLOCK_TOKENS] = id;
        }
        slot_mapping_out[b] =
            static_cast<int64_t>(row[c / KV_BLOCK_TOKENS]) * KV_BLOCK_TOKENS + c % KV_BLOCK_TOKENS;
        context_lens[b] = c + 1;
    }
    return KV_OK;
}

extern "C" kv_status kv_pool_fork(void *pool, const int32_t *parent_row, int n_blocks, int32_t *child_row)
{
    if (!pool || n_blocks < 0 || (n_blocks > 0 && (!parent_row || !child_row)))
        return KV_ERR_ARG;
    BlockPool *p = as_pool(pool);
    std::lock_guard<std::mutex> lock(p->mu);
    const int64_t nb = static_cast<int64_t>(p->refcount.size());
    for (int i = 0; i < n_blocks; ++i)
        if (parent_row[i] < 0 || parent_row[i] >= nb || p->refcount[static_cast<size_t>(parent_row[i])] <= 0)
            return KV_ERR_STATE;
    for (int i = 0; i < n_blocks; ++i) {
        ++p->refcount[static_cast<size_t>(parent_row[i])];
        child_row[i] = parent_row[i];
    }
    return KV_OK;
}

extern "C" kv_status kv_pool_append_slots_cow(void *pool, int32_t *block_tables, int W, int32_t *context_lens, int B,
                                              int64_t *slot_mapping_out, int32_t *copy_src_out,
                                              int32_t *copy_dst_out, int *n_copies_out)
{
    pkv_host::NvtxRange nvtx_range("kv_pool_append_slots_cow");
    if (!pool || B < 0 || W < 1 || !n_copies_out ||
        (B > 0 && (!block_tables || !context_lens || !slot_mapping_out || !copy_src_out || !copy_dst_out)))
        return KV_ERR_ARG;
    BlockPool *p = as_pool(pool);
    std::lock_guard<std::mutex> lock(p->mu);
    const int64_t nb = static_cast<int64_t>(p->refcount.size());
    // validate the whole step first; count fresh blocks and copies
    size_t need = 0;
    std::unordered_map<int32_t, int> drops;  // references the copies will give up, per shared block
    for (int b = 0; b < B; ++b) {
        const int c = context_lens[b];
        if (c < 0 || c / KV_BLOCK_TOKENS >= W)
            return KV_ERR_ARG;
        if (c % KV_BLOCK_TOKENS == 0) {
            ++need;
            continue;
        }
        const int32_t tail = block_tables[static_cast<size_t>(b) * W + c / KV_BLOCK_TOKENS];
        if (tail < 0 || tail >= nb || p->refcount[static_cast<size_t>(tail)] <= 0)
            return KV_ERR_STATE;
        if (p->refcount[static_cast<size_t>(tail)] > 1)
            ++drops[tail];
    }
    // A block whose every reference appends this step would be copied for all of
    // them and then freed; the last of them keeps it instead (it is then private).
    for (auto &kv : drops) {
        if (kv.second >= p->refcount[static_cast<size_t>(kv.first)])
            kv.second = p->refcount[static_cast<size_t>(kv.first)] - 1;
        need += static_cast<size_t>(kv.second);
    }
    if (need > p->free_ids.size())
        return KV_ERR_OOM;
    int copies = 0;
    for (int b = 0; b < B; ++b) {
        const int c = context_lens[b];
        int32_t *row = block_tables + static_cast<size_t>(b) * W;
        if (c % KV_BLOCK_TOKENS == 0) {
            const int32_t id = p->free_ids.back();
            p->free_ids.pop_back();
            p->refcount[static_cast<size_t>(id)] = 1;
            row[c / KV_BLOCK_TOKENS] = id;
        } else {
            const int32_t tail = row[c / KV_BLOCK_TOKENS];
            auto it = drops.find(tail);
            if (it != drops.end() && it->second > 0) {
                --it->second;
                const int32_t id = p->free_ids.back();
                p->free_ids.pop_back();
                p->refcount[static_cast<size_t>(id)] = 1;
                --p->refcount[static_cast<size_t>(tail)];
                row[c / KV_BLOCK_TOKENS] = id;
                copy_src_out[copies] = tail;
                copy_dst_out[copies] = id;
                ++copies;
            }
        }
        slot_mapping_out[b] =
            static_cast<int64_t>(row[c / KV_BLOCK_TOKENS]) * KV_BLOCK_TOKENS + c % KV_BLOCK_TOKENS;
        context_lens[b] = c + 1;
    }
    *n_copies_out = copies;
    return KV_OK;
}

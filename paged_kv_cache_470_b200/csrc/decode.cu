// paged_attention_decode: one decode step of grouped-query attention over a
// paged KV cache, for sm_100a.
//
// What is computed ("Module 23: Serving", sections 23.2 and 23.4; "Scaling LLM
// serving", section "The KV cache"): for sequence b with c cached tokens and
// query head h, with kv head j = h / (Hq / Hkv),
//     out[b][h] = sum_t softmax_t(scale * <q[b][h], K_t>) V_t,   t < c,
// where token t lives in physical block block_tables[b][t / 16], row t % 16.
//
// Work decomposition. The kv heads are taken in groups of HG (4 when Hkv is a
// multiple of 4, else 2 or 1). A work item is (sequence b, kv-head group,
// chunk of at most 8 query heads per kv head); its work units are the
// ceil(c/16) KV blocks of the sequence, each unit being the group's HG heads of
// one block: one TMA box of 16 rows x HG heads x 64 columns (8 KB when HG=4)
// per 64 columns of K and of V. A box costs about as much to issue as one four
// times larger, so HG heads travel together.
//
// All units of all items are laid end to end and cut into equal contiguous
// ranges, one per CTA (one resident CTA per SM). A CTA handles whole items
// and at most two partial ones; an item cut between CTAs is a split-K item:
// each piece leaves (running max, running sum, unnormalised accumulator) in
// fp32 and a log-sum-exp merge joins them, in the last CTA to finish a piece
// of that item (an atomic counter, no spinning) or in a separate combine
// kernel.
//
// Inside a CTA, warp 8 is the producer: it reads block ids from the table and
// issues the TMA loads into a ring of shared-memory stages guarded by
// mbarriers. Warps 0-7 are consumers arranged as 8/HG streams of HG warps:
// stream s takes units s, s + 8/HG, ...; within a stream, warp hh handles kv
// head hh of the group. Each warp keeps an fp32 online softmax (running max
// and sum per query head) and its accumulator in registers; at the end of an
// item the streams are merged pairwise through shared memory.
//
// Two consumer arithmetic paths:
//  * tensor cores: S^T[16 tokens x 8 heads] = K_blk * Q^T with
//    mma.sync.m16n8k16 (16-bit in, fp32 accumulate; the 16 tokens of a block are
//    the M dimension, the kv head's query heads the N dimension), then
//    O^T[D x 8] += V_blk^T * P^T, with the probabilities split into a 16-bit
//    high part and a 16-bit residual so that P keeps ~16 (bf16) or ~22 (fp16)
//    significant bits.
//  * CUDA cores: fp32 FMAs on values unpacked from 16 bits.
//
// q, the cache and out are all bf16 or all fp16 (the element type E); the
// cache holds 2 bytes per number either way ("Module 23: Serving", section
// 23.1).
//
// Layers. One launch may cover L layers of one decode step ("Module 23:
// Serving", section 23.1: every layer holds its own K and V for every token):
// q, out and the new token rows are stacked [L][B][...], the caches are L
// equally shaped pools a fixed stride apart, and the block tables and lengths
// are shared by all layers (a sequence's position -> block map does not depend
// on the layer). The work positions of layer l follow those of layer l - 1, so
// the split-K tail of one layer overlaps the next layer's streaming; L = 1 is
// the per-layer call.
#include "pkv_device.cuh"
#include "nvtx_range.h"
#include "pagedkv.h"
#include "tma_host.h"

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

namespace pkv {

constexpr int kConsumerWarps = 8;
constexpr int kConsumerThreads = kConsumerWarps * 32;
constexpr int kProducerWarp = kConsumerWarps;
constexpr int kHelperWarp = kConsumerWarps + 1;   // counts finished split pieces off the consumers' path
constexpr int kThreads = kConsumerThreads + 64;
constexpr int kPieceQueue = 4;                    // consumer -> helper queue of finished split pieces
constexpr int kBarConsumers = 1;                  // named barrier of the consumer warps
constexpr int kGroupMax = 8;            // query heads per kv head per work item
constexpr int kMaxHG = 4;               // kv heads per work unit
constexpr int kHeadTileBytes = 2048;    // one kv head: 16 rows x 64 elements, 128B-swizzled
constexpr int kMergeSlots = 4;          // warps that hand their state over per merge round
constexpr int kCtasPerSm = 1;
constexpr int kStatusBytes = 256;
constexpr unsigned kFull = 0xffffffffu;

enum ComputePath { kPathMma = 1, kPathSimt = 2 };
constexpr int kMergeBatch = 4;          // split-K pieces whose loads are in flight together

constexpr int cmax(int a, int b) { return a > b ? a : b; }

template <int D>
struct Geo {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kTiles = D / 64;                       // 64-column boxes per K (and per V)
    static constexpr int kRingBytes = 192 * 1024;
    static constexpr int kMaxStages = kRingBytes / (2 * kTiles * kHeadTileBytes);  // HG = 1
    static constexpr int kMmaRegs = (D / 16) * 4 + 4;
    static constexpr int kSimtRegs = kGroupMax * (D / 32) + 2 * kGroupMax;
    static constexpr int kMergeBytes = kMergeSlots * cmax(kMmaRegs, kSimtRegs) * 32 * 4;
    static constexpr int kQStride = D + 8;                      // second half shifted by 4 floats
    static constexpr int kQBytes = kMaxHG * kGroupMax * kQStride * 4;
    static constexpr int kPBytes = kConsumerWarps * 16 * kGroupMax * 4;
    static constexpr int kOwnBytes = kMaxHG * kGroupMax * (D + 2) * 4;  // a piece's state, for the solo merge
    static constexpr int kScratchBytes = cmax(cmax(kMergeBytes, kQBytes + kPBytes), kOwnBytes);
    static constexpr int kOffScratch = kRingBytes;
    static constexpr int kOffBar = kOffScratch + kScratchBytes;
    static constexpr int kOffQBar = kOffBar + 2 * kMaxStages * 8;    // piece queue: full[4], empty[4]
    static constexpr int kOffMisc = kOffQBar + 2 * kPieceQueue * 8;
    static constexpr int kMiscInts = 64;
    static constexpr int kSmemBytes = kOffMisc + kMiscInts * 4 + 1024;  // + room to align the base
};

struct DecodeArgs {
    uint16_t *out;        // [L][B][Hq][D] elements of type E (fp32 numbers when out_f32)
    const uint16_t *q;    // [L][B][Hq][D]
    const int32_t *block_tables;
    const int32_t *context_lens;
    float *part_acc;     // [slots][kMaxHG][8][D]
    float *part_ml;      // [slots][kMaxHG][8][2]  (max in log2 units, sum)
    int32_t *counters;   // [items]
    int32_t *status;
    int B, W, Hq, Hkv, group, num_blocks;
    int L;               // layers in this launch
    int out_f32;         // out holds fp32 numbers (a debug switch: the result before rounding)
    int hg;              // kv heads per unit (HG)
    int streams;         // consumer streams = 8 / HG
    int hchunks;         // query-head chunks per kv head = ceil(group / 8)
    int items_per_seq;   // (Hkv / HG) * hchunks
    int stages, stage_bytes, tile_stride;  // ring geometry; tile_stride = HG * 2048
    int prod_lanes;      // producer lanes issuing TMA
    int min_chunk;
    int item_cost;       // work positions charged per work item on top of its units
    int drop_unit;       // test hook: the CTA holding the launch's first unit never loads its unit with
                         // this index (-1: none)
    int l2_policy;       // L2 priority of the K/V tile loads: 1 evict first, 2 evict normal, 3 evict last
    int early_loads;     // issue the first ring of tile loads before the grid dependency wait (caller's promise)
    int fused;
    float scale_log2;    // scale * log2(e)
    // fused append (append != 0): this step's token of sequence b is k_new/v_new[b],
    // at slot slots[b], which must be position context_lens[b] - 1 of sequence b
    int append;
    const uint4 *k_new, *v_new;   // [L][B][Hkv][D], as 16-byte chunks
    uint4 *k_cache, *v_cache;     // layer 0's [num_blocks][16][Hkv][D], as 16-byte chunks
    size_t cache_layer_chunks;    // 16-byte chunks from one layer's cache to the next
    const int64_t *slots;         // [B], shared by the layers
};

// misc ints in shared memory
enum {
    kMiscAbort = 0,
    kMiscLocB = 1,
    kMiscSolo = 3,      // this piece's item has all its other pieces finished
    kMiscZero = 4,
    kMiscLast = 5,      // the CTA's final piece completed its item: merge it
    kMiscQueue = 16,    // kPieceQueue descriptors of 5 ints: item, first cta, last cta, b, k
    kMiscLocK = 36,     // item and block offset of the CTA's first unit (sequence in kMiscLocB)
    kMiscLocOff = 37,
    kMiscLocPos = 38,   // work position of that item's first unit
    kMiscStartU = 39,   // units before the CTA's range, and before its end
    kMiscEndU = 40,
    kMiscEndFound = 41,
    kMiscLocLayer = 42, // layer of the CTA's first unit
    kMiscStartFound = 43,
    kMiscScan64 = 44,   // 10 64-bit warp sums (ints 44..63)
};

__device__ __forceinline__ int clamp_ctx(int c, int W)
{
    return c < 0 ? 0 : (c > W * kBlockTokens ? W * kBlockTokens : c);
}
__device__ __forceinline__ int seq_ctx(const DecodeArgs &a, int b) { return clamp_ctx(__ldg(a.context_lens + b), a.W); }
__device__ __forceinline__ int ctx_blocks(int c) { return (c + kBlockTokens - 1) / kBlockTokens; }

// Inclusive scan over all kThreads threads; *total receives the sum.
__device__ __forceinline__ long long block_scan_incl64(long long v, volatile long long *warp_sums, long long *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long y = __shfl_up_sync(kFull, x, o);
        if (lane >= o)
            x += y;
    }
    if (lane == 31)
        warp_sums[warp] = x;
    __syncthreads();
    long long pre = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) {
        const long long s = warp_sums[w];
        pre += (w < warp) ? s : 0;
        tot += s;
    }
    __syncthreads();
    *total = tot;
    return x + pre;
}

// Work positions. The units of all items are laid end to end, and each item of
// a non-empty sequence is preceded by a.item_cost positions that stand for its
// fixed cost (query loads, the merge of the consumer streams, the store or the
// split-K hand-off). CTAs take equal ranges of positions, so a CTA that starts
// more items gets fewer units. Per sequence, the scan carries
// (positions << 24) + (1 if the sequence has blocks).
constexpr int kNonEmptyBits = 24;
__device__ __forceinline__ long long seq_scan_value(const DecodeArgs &a, int n)
{
    return n > 0 ? ((static_cast<long long>(a.items_per_seq) * (n + a.item_cost)) << kNonEmptyBits) + 1 : 0;
}

struct Cursor {
    int layer; // layer
    int b;     // sequence
    int k;     // item within the sequence: head group * hchunks + query-head chunk
    int off;   // block offset within the sequence
    int ctx;   // tokens of sequence b (clamped)
    int n;     // blocks of sequence b
    int pos;   // work position of the item's first unit
};

__device__ __forceinline__ void cursor_next_item(const DecodeArgs &a, Cursor &c)
{
    c.pos += c.n + a.item_cost;
    c.off = 0;
    if (++c.k == a.items_per_seq) {
        c.k = 0;
        for (;;) {
            if (++c.b == a.B) {
                if (c.layer + 1 == a.L) {  // past the last item of the launch
                    c.ctx = c.n = 0;
                    break;
                }
                ++c.layer;  // the next layer starts again at the first sequence
                c.b = 0;
            }
            c.ctx = seq_ctx(a, c.b);
            c.n = ctx_blocks(c.ctx);
            if (c.n > 0)
                break;
        }
    }
}

__device__ __forceinline__ uint4 lds128(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint2 lds64(uint32_t addr)
{
    uint2 v;
    asm volatile("ld.shared.v2.b32 {%0,%1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(addr));
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr)
{
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
    return v;
}
__device__ __forceinline__ void sts128_zero(uint32_t addr)
{
    asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(addr), "r"(0) : "memory");
}

// Byte offset of 16-byte chunk `chunk` (0..7) of row `row` inside one head's 128B-swizzled tile.
__device__ __forceinline__ uint32_t swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

// Split-K counters. A finished piece is counted in with an acq_rel atomic (the
// writes of its other threads are ordered before it by a bar.sync); the one
// whose count completes the item has, by the same atomic, acquired the other
// pieces' partials. A CTA that sees a complete count by a relaxed load (read
// early, so the load's round trip is hidden) issues an acquire fence before
// merging.
__device__ __forceinline__ int ld_relaxed_gpu(const int32_t *p)
{
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ int atom_add_acq_rel_gpu(int32_t *p, int v)
{
    int prev;
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(prev) : "l"(p), "r"(v) : "memory");
    return prev;
}
__device__ __forceinline__ void fence_acquire_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// exp2(x - m) for merging states whose maxima may both be -inf (empty states).
__device__ __forceinline__ float rescale(float x, float m) { return m == -INFINITY ? 0.f : exp2f(x - m); }

// The new token of one kv head of an item, for the fused append: lane l < D/8
// holds 16-byte chunk l of the K row, lane D/8 <= l < D/4 chunk l - D/8 of the
// V row. `slot` is where it goes (-1: nothing to append, or a bad slot) and
// `dst` the index of its first 16-byte chunk in the layer's K (or V) cache.
struct AppendRow {
    uint4 chunk;
    long long slot;
    size_t dst;
};

// Row (layer, sequence) of q and out: layer * B + b.
__device__ __forceinline__ int layer_row(const DecodeArgs &a, const Cursor &cur) { return cur.layer * a.B + cur.b; }

// Work item index within the launch: (layer * B + b) * items_per_seq + k.
__device__ __forceinline__ int item_index(const DecodeArgs &a, const Cursor &cur)
{
    return layer_row(a, cur) * a.items_per_seq + cur.k;
}

// Where an item's outputs go.
struct ItemOut {
    int lb, h0, gc;  // row (layer, sequence) of q and out, first query head of this warp's kv head,
                     // valid query heads (<= 8)
    size_t slot;     // split-K piece slot (only for partial items)
    int hh;          // kv head within the group
};

__device__ __forceinline__ ItemOut item_out(const DecodeArgs &a, const Cursor &cur, int hh)
{
    const int hg = cur.k / a.hchunks, hc = cur.k - hg * a.hchunks;
    ItemOut o;
    o.lb = layer_row(a, cur);
    o.hh = hh;
    o.h0 = (hg * a.hg + hh) * a.group + hc * kGroupMax;
    o.gc = min(kGroupMax, a.group - hc * kGroupMax);
    o.slot = static_cast<size_t>(blockIdx.x) + static_cast<size_t>(item_index(a, cur));
    return o;
}

// One output number at element index i of out (element type E, or fp32 when out_f32).
template <class E>
__device__ __forceinline__ void put_out(const DecodeArgs &a, size_t i, float v)
{
    if (a.out_f32)
        reinterpret_cast<float *>(a.out)[i] = v;
    else
        a.out[i] = E::from_f32(v);
}

// ---------------------------------------------------------------------------
// Per-warp consumer state and arithmetic (one kv head of each unit).
// ---------------------------------------------------------------------------
template <class E, int D, int PATH, int NH>
struct Consumer;

// Tensor-core path. Lane (r = lane/4, c = lane%4) holds scores of tokens r and
// r+8 for query heads 2c and 2c+1, and the accumulator O^T rows d = 16*mt + r
// (+8) for the same two heads.
template <class E, int D, int NH>
struct Consumer<E, D, kPathMma, NH> {
    static constexpr int kTiles = D / 64;
    static constexpr int kMt = D / 16;
    static constexpr int kRegs = kMt * 4 + 4;
    uint32_t qf[kMt][2];   // this item's query fragments (B operand of S^T = K Q^T)
    uint32_t qn[kMt][2];   // the next item's, loaded one item ahead
    float acc[kMt][4];
    float m0, m1, l0, l1;

    // Issue the loads of an item's query fragments into qn (used at its begin_item).
    __device__ __forceinline__ void prefetch_q(const DecodeArgs &a, const ItemOut &o)
    {
        const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
        const uint32_t *qrow =
            reinterpret_cast<const uint32_t *>(a.q + (static_cast<size_t>(o.lb) * a.Hq + o.h0 + r) * D);
#pragma unroll
        for (int kk = 0; kk < kMt; ++kk) {
            qn[kk][0] = (r < o.gc) ? __ldg(qrow + kk * 8 + c) : 0u;
            qn[kk][1] = (r < o.gc) ? __ldg(qrow + kk * 8 + 4 + c) : 0u;
        }
    }

    __device__ __forceinline__ void begin_item(const DecodeArgs &, const ItemOut &, const float *)
    {
#pragma unroll
        for (int kk = 0; kk < kMt; ++kk) {
            qf[kk][0] = qn[kk][0];
            qf[kk][1] = qn[kk][1];
        }
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt)
            acc[mt][0] = acc[mt][1] = acc[mt][2] = acc[mt][3] = 0.f;
        m0 = m1 = -INFINITY;
        l0 = l1 = 0.f;
    }

    __device__ __forceinline__ void unit(uint32_t kbase, uint32_t vbase, int tile_stride, int valid, float sl2,
                                         const float *, float *)
    {
        const int lane = threadIdx.x & 31, r = lane >> 2, mi = lane >> 3, rr = lane & 7;
        if (valid < 16) {
            // rows past the context hold whatever the pool holds; zero them so 0 * V stays 0
            const int rows = 16 - valid;
            for (int idx = lane; idx < rows * 8 * kTiles; idx += 32) {
                const int t = idx / (8 * kTiles);
                const int rem = idx - t * 8 * kTiles;
                const int tile = rem >> 3, ch = rem & 7;
                sts128_zero(vbase + tile * tile_stride + (valid + t) * 128 + ch * 16);
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            __syncwarp();
        }
        // S^T = K_blk [16 x D] * Q^T [D x 8]
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const int row = ((mi & 1) << 3) + rr;
#pragma unroll
            for (int kk = 0; kk < kMt; ++kk) {
                const int tile = kk >> 2, kc = kk & 3;
                uint32_t af[4];
                ldmatrix_x4(af, kbase + tile * tile_stride + swz(row, (kc << 1) + (mi >> 1)));
                E::mma(s, af, qf[kk][0], qf[kk][1]);
            }
        }
        const bool v0 = r < valid, v1 = (r + 8) < valid;
        const float s0 = v0 ? s[0] * sl2 : -INFINITY;
        const float s1 = v0 ? s[1] * sl2 : -INFINITY;
        const float s2 = v1 ? s[2] * sl2 : -INFINITY;
        const float s3 = v1 ? s[3] * sl2 : -INFINITY;
        float bm0 = fmaxf(s0, s2), bm1 = fmaxf(s1, s3);
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            bm0 = fmaxf(bm0, __shfl_xor_sync(kFull, bm0, o));
            bm1 = fmaxf(bm1, __shfl_xor_sync(kFull, bm1, o));
        }
        const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
        const float al0 = exp2f(m0 - mn0), al1 = exp2f(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        const float p0 = exp2f(s0 - mn0), p1 = exp2f(s1 - mn1);
        const float p2 = exp2f(s2 - mn0), p3 = exp2f(s3 - mn1);
        l0 = l0 * al0 + (p0 + p2);
        l1 = l1 * al1 + (p1 + p3);
        // P^T as a 16-bit high part plus a 16-bit residual, transposed into B fragments
        const uint32_t h01 = E::pack(p0, p1), h23 = E::pack(p2, p3);
        const uint32_t r01 = E::pack(p0 - E::lo(h01), p1 - E::hi(h01));
        const uint32_t r23 = E::pack(p2 - E::lo(h23), p3 - E::hi(h23));
        const uint32_t bh0 = movmatrix_trans(h01), bh1 = movmatrix_trans(h23);
        const uint32_t bl0 = movmatrix_trans(r01), bl1 = movmatrix_trans(r23);
        // O^T [D x 8] += V_blk^T [D x 16] * P^T [16 x 8]
        const int vrow = ((mi >> 1) << 3) + rr;
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) {
            acc[mt][0] *= al0;
            acc[mt][1] *= al1;
            acc[mt][2] *= al0;
            acc[mt][3] *= al1;
            const int tile = mt >> 2, kc = mt & 3;
            uint32_t af[4];
            ldmatrix_x4_trans(af, vbase + tile * tile_stride + swz(vrow, (kc << 1) + (mi & 1)));
            E::mma(acc[mt], af, bh0, bh1);
            E::mma(acc[mt], af, bl0, bl1);
        }
    }

    // Sum the running sums over the lanes that share a query head.
    __device__ __forceinline__ void finish()
    {
#pragma unroll
        for (int o = 4; o < 32; o <<= 1) {
            l0 += __shfl_xor_sync(kFull, l0, o);
            l1 += __shfl_xor_sync(kFull, l1, o);
        }
    }

    // Hand this warp's state to a partner warp (same kv head, same lane layout).
    __device__ __forceinline__ void save(float *slot) const
    {
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt)
#pragma unroll
            for (int i = 0; i < 4; ++i)
                slot[(mt * 4 + i) * 32 + lane] = acc[mt][i];
        slot[(kMt * 4 + 0) * 32 + lane] = m0;
        slot[(kMt * 4 + 1) * 32 + lane] = m1;
        slot[(kMt * 4 + 2) * 32 + lane] = l0;
        slot[(kMt * 4 + 3) * 32 + lane] = l1;
    }

    __device__ __forceinline__ void merge(const float *slot)
    {
        const int lane = threadIdx.x & 31;
        const float pm0 = slot[(kMt * 4 + 0) * 32 + lane], pm1 = slot[(kMt * 4 + 1) * 32 + lane];
        const float pl0 = slot[(kMt * 4 + 2) * 32 + lane], pl1 = slot[(kMt * 4 + 3) * 32 + lane];
        const float M0 = fmaxf(m0, pm0), M1 = fmaxf(m1, pm1);
        const float a0 = rescale(m0, M0), b0 = rescale(pm0, M0);
        const float a1 = rescale(m1, M1), b1 = rescale(pm1, M1);
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) {
            acc[mt][0] = acc[mt][0] * a0 + slot[(mt * 4 + 0) * 32 + lane] * b0;
            acc[mt][1] = acc[mt][1] * a1 + slot[(mt * 4 + 1) * 32 + lane] * b1;
            acc[mt][2] = acc[mt][2] * a0 + slot[(mt * 4 + 2) * 32 + lane] * b0;
            acc[mt][3] = acc[mt][3] * a1 + slot[(mt * 4 + 3) * 32 + lane] * b1;
        }
        l0 = l0 * a0 + pl0 * b0;
        l1 = l1 * a1 + pl1 * b1;
        m0 = M0;
        m1 = M1;
    }

    __device__ __forceinline__ void store_final(const DecodeArgs &a, const ItemOut &o) const
    {
        const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
        const int n0 = 2 * c, n1 = 2 * c + 1;
        const float i0 = 1.f / l0, i1 = 1.f / l1;
        const size_t o0 = (static_cast<size_t>(o.lb) * a.Hq + o.h0 + n0) * D;
        const size_t o1 = o0 + D;
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) {
            const int d = mt * 16 + r;
            if (n0 < o.gc) {
                put_out<E>(a, o0 + d, acc[mt][0] * i0);
                put_out<E>(a, o0 + d + 8, acc[mt][2] * i0);
            }
            if (n1 < o.gc) {
                put_out<E>(a, o1 + d, acc[mt][1] * i1);
                put_out<E>(a, o1 + d + 8, acc[mt][3] * i1);
            }
        }
    }

    // This warp's unnormalised state for its kv head, in the piece layout
    // [kv head][query head][D] and [kv head][query head][2] starting at
    // part_acc / part_ml (a global slot, or the CTA's own copy in shared memory).
    __device__ __forceinline__ void store_state(const ItemOut &o, float *part_acc, float *part_ml) const
    {
        const int lane = threadIdx.x & 31, r = lane >> 2, c = lane & 3;
        const int n0 = 2 * c, n1 = 2 * c + 1;
        const size_t head0 = static_cast<size_t>(o.hh) * kGroupMax;
        float *p0 = part_acc + (head0 + n0) * D;
        float *p1 = part_acc + (head0 + n1) * D;
#pragma unroll
        for (int mt = 0; mt < kMt; ++mt) {
            const int d = mt * 16 + r;
            if (n0 < o.gc) {
                p0[d] = acc[mt][0];
                p0[d + 8] = acc[mt][2];
            }
            if (n1 < o.gc) {
                p1[d] = acc[mt][1];
                p1[d + 8] = acc[mt][3];
            }
        }
        if (r == 0) {
            if (n0 < o.gc) {
                part_ml[(head0 + n0) * 2] = m0;
                part_ml[(head0 + n0) * 2 + 1] = l0;
            }
            if (n1 < o.gc) {
                part_ml[(head0 + n1) * 2] = m1;
                part_ml[(head0 + n1) * 2 + 1] = l1;
            }
        }
    }
};

// CUDA-core path. QK: lane (t = lane/2, half = lane%2) dots token t's half row
// with every query head; PV: lane owns D/32 output columns for every head.
template <class E, int D, int NH>
struct Consumer<E, D, kPathSimt, NH> {
    static constexpr int C = D / 32;     // output columns per lane
    static constexpr int CPH = D / 16;
    static constexpr int kRegs = NH * C + 2 * NH;
    float acc[NH][C];
    float m[NH], l[NH];

    // The CUDA-core path stages the whole item's q in shared memory instead.
    __device__ __forceinline__ void prefetch_q(const DecodeArgs &, const ItemOut &) {}

    __device__ __forceinline__ void begin_item(const DecodeArgs &, const ItemOut &, const float *)
    {
#pragma unroll
        for (int n = 0; n < NH; ++n) {
#pragma unroll
            for (int e = 0; e < C; ++e)
                acc[n][e] = 0.f;
            m[n] = -INFINITY;
            l[n] = 0.f;
        }
    }

    // q_s: this kv head's [8][kQStride] fp32 rows; p_s: this warp's [16][8] fp32
    __device__ __forceinline__ void unit(uint32_t kbase, uint32_t vbase, int tile_stride, int valid, float sl2,
                                         const float *q_s, float *p_s)
    {
        constexpr int QS = Geo<D>::kQStride;
        const int lane = threadIdx.x & 31, t = lane >> 1, half = lane & 1;
        float dot[NH];
#pragma unroll
        for (int n = 0; n < NH; ++n)
            dot[n] = 0.f;
#pragma unroll
        for (int cc = 0; cc < CPH; ++cc) {
            const int dcol = half * (D / 2) + cc * 8;
            const uint4 kv = lds128(kbase + (dcol >> 6) * tile_stride + swz(t, (dcol & 63) >> 3));
            const float k0 = E::lo(kv.x), k1 = E::hi(kv.x), k2 = E::lo(kv.y), k3 = E::hi(kv.y),
                        k4 = E::lo(kv.z), k5 = E::hi(kv.z), k6 = E::lo(kv.w), k7 = E::hi(kv.w);
            const float *qs = q_s + dcol + half * 4;
#pragma unroll
            for (int n = 0; n < NH; ++n) {
                const float4 qa = *reinterpret_cast<const float4 *>(qs + n * QS);
                const float4 qb = *reinterpret_cast<const float4 *>(qs + n * QS + 4);
                float x = dot[n];
                x = fmaf(k0, qa.x, x);
                x = fmaf(k1, qa.y, x);
                x = fmaf(k2, qa.z, x);
                x = fmaf(k3, qa.w, x);
                x = fmaf(k4, qb.x, x);
                x = fmaf(k5, qb.y, x);
                x = fmaf(k6, qb.z, x);
                x = fmaf(k7, qb.w, x);
                dot[n] = x;
            }
        }
        float al[NH];
#pragma unroll
        for (int n = 0; n < NH; ++n) {
            const float full_dot = dot[n] + __shfl_xor_sync(kFull, dot[n], 1);
            const float sv = (t < valid) ? full_dot * sl2 : -INFINITY;
            float bm = sv;
#pragma unroll
            for (int o = 2; o < 32; o <<= 1)
                bm = fmaxf(bm, __shfl_xor_sync(kFull, bm, o));
            const float mn = fmaxf(m[n], bm);
            al[n] = exp2f(m[n] - mn);
            m[n] = mn;
            const float p = exp2f(sv - mn);
            l[n] = l[n] * al[n] + p;
            if (half == 0)
                p_s[t * kGroupMax + n] = p;
        }
        __syncwarp();
        const int d0 = lane * C;
        const uint32_t vcol = (d0 >> 6) * tile_stride;
        const int chunk = (d0 & 63) >> 3, within = d0 & 7;
#pragma unroll
        for (int n = 0; n < NH; ++n)
#pragma unroll
            for (int e = 0; e < C; ++e)
                acc[n][e] *= al[n];
        for (int tt = 0; tt < valid; ++tt) {
            const uint32_t addr = vbase + vcol + swz(tt, chunk) + within * 2;
            float v[C];
            if constexpr (C == 4) {
                const uint2 w = lds64(addr);
                v[0] = E::lo(w.x);
                v[1] = E::hi(w.x);
                v[2] = E::lo(w.y);
                v[3] = E::hi(w.y);
            } else {
                const uint32_t w = lds32(addr);
                v[0] = E::lo(w);
                v[1] = E::hi(w);
            }
            const float *pr = p_s + tt * kGroupMax;
#pragma unroll
            for (int n = 0; n < NH; ++n) {
                const float pn = pr[n];
#pragma unroll
                for (int e = 0; e < C; ++e)
                    acc[n][e] = fmaf(pn, v[e], acc[n][e]);
            }
        }
        __syncwarp();
    }

    __device__ __forceinline__ void finish()
    {
#pragma unroll
        for (int n = 0; n < NH; ++n)
#pragma unroll
            for (int o = 2; o < 32; o <<= 1)
                l[n] += __shfl_xor_sync(kFull, l[n], o);
    }

    __device__ __forceinline__ void save(float *slot) const
    {
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int n = 0; n < NH; ++n) {
#pragma unroll
            for (int e = 0; e < C; ++e)
                slot[(n * C + e) * 32 + lane] = acc[n][e];
            slot[(NH * C + n) * 32 + lane] = m[n];
            slot[(NH * C + NH + n) * 32 + lane] = l[n];
        }
    }

    __device__ __forceinline__ void merge(const float *slot)
    {
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int n = 0; n < NH; ++n) {
            const float pm = slot[(NH * C + n) * 32 + lane], pl = slot[(NH * C + NH + n) * 32 + lane];
            const float M = fmaxf(m[n], pm);
            const float a = rescale(m[n], M), b = rescale(pm, M);
#pragma unroll
            for (int e = 0; e < C; ++e)
                acc[n][e] = acc[n][e] * a + slot[(n * C + e) * 32 + lane] * b;
            l[n] = l[n] * a + pl * b;
            m[n] = M;
        }
    }

    __device__ __forceinline__ void store_final(const DecodeArgs &a, const ItemOut &o) const
    {
        const int lane = threadIdx.x & 31;
#pragma unroll
        for (int n = 0; n < NH; ++n) {
            if (n < o.gc) {
                const float inv = 1.f / l[n];
                const size_t dst = (static_cast<size_t>(o.lb) * a.Hq + o.h0 + n) * D + lane * C;
#pragma unroll
                for (int e = 0; e < C; ++e)
                    put_out<E>(a, dst + e, acc[n][e] * inv);
            }
        }
    }

    __device__ __forceinline__ void store_state(const ItemOut &o, float *part_acc, float *part_ml) const
    {
        const int lane = threadIdx.x & 31;
        const size_t head0 = static_cast<size_t>(o.hh) * kGroupMax;
#pragma unroll
        for (int n = 0; n < NH; ++n) {
            if (n < o.gc) {
                float *dst = part_acc + (head0 + n) * D + lane * C;
#pragma unroll
                for (int e = 0; e < C; ++e)
                    dst[e] = acc[n][e];
                if (lane == 0) {
                    part_ml[(head0 + n) * 2] = m[n];
                    part_ml[(head0 + n) * 2 + 1] = l[n];
                }
            }
        }
    }
};

// Log-sum-exp merge of the split-K pieces of one item. The item's pieces sit in
// slots first_cta + item .. last_cta + item of the workspace, except that piece
// `own_cta` (if own_acc is not null) is read from the caller's shared-memory
// copy in the same layout. A thread takes NC consecutive groups of four output
// columns of one (kv head, query head) row, and issues all loads for MB pieces
// before using any, so a merge costs about one memory round trip per MB pieces.
// The order of the arithmetic depends only on the pieces, not on which CTA
// merges.
template <class E, int D>
__device__ __forceinline__ void merge_pieces_global(const DecodeArgs &a, int item, int first_cta, int last_cta,
                                                    int lb, int k, int tid, int nthreads, int own_cta = -1,
                                                    const float *own_acc = nullptr, const float *own_ml = nullptr)
{
    constexpr int NC = D == 128 ? 4 : 2;          // float4 column groups per thread
    constexpr int MB = D == 128 ? 2 : kMergeBatch;  // pieces per round of loads
    constexpr int TPR = D / 4 / NC;               // threads per row
    const int hg = k / a.hchunks, hc = k - hg * a.hchunks;
    const int gc = min(kGroupMax, a.group - hc * kGroupMax);
    const int rows = a.hg * gc;
    const int rows_per_pass = nthreads / TPR;
    for (int row = tid / TPR; row < rows; row += rows_per_pass) {
        if (tid >= rows_per_pass * TPR)
            break;
        const int hh = row / gc, n = row - hh * gc;
        const int head = hh * kGroupMax + n;      // within a slot
        const int col0 = (tid % TPR) * NC * 4;
        float M = -INFINITY, L = 0.f;
        float4 O[NC];
#pragma unroll
        for (int e = 0; e < NC; ++e)
            O[e] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int c0 = first_cta; c0 <= last_cta; c0 += MB) {
            float mv[MB], lv[MB];
            float4 ov[MB][NC];
#pragma unroll
            for (int j = 0; j < MB; ++j) {
                const int c = c0 + j;
                if (c > last_cta) {
                    mv[j] = -INFINITY;
                    lv[j] = 0.f;
#pragma unroll
                    for (int e = 0; e < NC; ++e)
                        ov[j][e] = make_float4(0.f, 0.f, 0.f, 0.f);
                } else if (c == own_cta && own_acc != nullptr) {
                    mv[j] = own_ml[head * 2];
                    lv[j] = own_ml[head * 2 + 1];
#pragma unroll
                    for (int e = 0; e < NC; ++e)
                        ov[j][e] = *reinterpret_cast<const float4 *>(own_acc + head * D + col0 + e * 4);
                } else {
                    const size_t h = (static_cast<size_t>(c) + item) * (kMaxHG * kGroupMax) + head;
                    mv[j] = __ldcg(a.part_ml + h * 2);
                    lv[j] = __ldcg(a.part_ml + h * 2 + 1);
#pragma unroll
                    for (int e = 0; e < NC; ++e)
                        ov[j][e] = __ldcg(reinterpret_cast<const float4 *>(a.part_acc + h * D + col0 + e * 4));
                }
            }
            float Mb = M;
#pragma unroll
            for (int j = 0; j < MB; ++j)
                Mb = fmaxf(Mb, mv[j]);
            const float sc = rescale(M, Mb);
            L *= sc;
#pragma unroll
            for (int e = 0; e < NC; ++e) {
                O[e].x *= sc;
                O[e].y *= sc;
                O[e].z *= sc;
                O[e].w *= sc;
            }
#pragma unroll
            for (int j = 0; j < MB; ++j) {
                const float w = rescale(mv[j], Mb);
                L = fmaf(w, lv[j], L);
#pragma unroll
                for (int e = 0; e < NC; ++e) {
                    O[e].x = fmaf(w, ov[j][e].x, O[e].x);
                    O[e].y = fmaf(w, ov[j][e].y, O[e].y);
                    O[e].z = fmaf(w, ov[j][e].z, O[e].z);
                    O[e].w = fmaf(w, ov[j][e].w, O[e].w);
                }
            }
            M = Mb;
        }
        const int h = (hg * a.hg + hh) * a.group + hc * kGroupMax + n;
        const float inv = 1.f / L;
        const size_t dst = (static_cast<size_t>(lb) * a.Hq + h) * D + col0;
#pragma unroll
        for (int e = 0; e < NC; ++e) {
            if (a.out_f32) {
                *reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.out) + dst + e * 4) =
                    make_float4(O[e].x * inv, O[e].y * inv, O[e].z * inv, O[e].w * inv);
            } else {
                uint2 packed;
                packed.x = E::pack(O[e].x * inv, O[e].y * inv);
                packed.y = E::pack(O[e].z * inv, O[e].w * inv);
                *reinterpret_cast<uint2 *>(a.out + dst + e * 4) = packed;
            }
        }
    }
}

// Load the new token row of kv head `j` of sequence b (fused append). The slot
// must be the sequence's last position; otherwise nothing is appended for it and
// KV_STATUS_BAD_SLOT is raised (by the first kv head's warp).
template <int D>
__device__ __forceinline__ AppendRow load_append_row(const DecodeArgs &a, const Cursor &cur, int j, bool report)
{
    AppendRow r;
    r.slot = -1;
    r.chunk = make_uint4(0u, 0u, 0u, 0u);
    if (!a.append || cur.ctx == 0)
        return r;
    const int lane = threadIdx.x & 31;
    const long long slot = __ldg(a.slots + cur.b);
    if (slot < 0)
        return r;
    const int last = cur.ctx - 1;
    const int blk = __ldg(a.block_tables + static_cast<size_t>(cur.b) * a.W + last / kBlockTokens);
    const long long expect = static_cast<long long>(blk) * kBlockTokens + last % kBlockTokens;
    if (slot != expect || blk < 0 || blk >= a.num_blocks) {
        if (report && lane == 0 && cur.layer == 0)  // every layer sees the same slot: report it once
            atomicOr(a.status, KV_STATUS_BAD_SLOT);
        return r;
    }
    r.slot = slot;
    constexpr int C = D / 8;  // 16-byte chunks per head row
    r.dst = cur.layer * a.cache_layer_chunks + (static_cast<size_t>(slot) * a.Hkv + j) * C;
    const size_t row = (static_cast<size_t>(layer_row(a, cur)) * a.Hkv + j) * C;
    if (lane < C)
        r.chunk = __ldg(a.k_new + row + lane);
    else if (lane < 2 * C)
        r.chunk = __ldg(a.v_new + row + lane - C);
    return r;
}

// Put the new token into this warp's tiles of the stage (row (c-1) % 16) and,
// if `write`, into the cache in global memory.
template <int D>
__device__ __forceinline__ void apply_append_row(const DecodeArgs &a, const AppendRow &r, int j, int row,
                                                 uint32_t kbase, uint32_t vbase, int tile_stride, bool write)
{
    constexpr int C = D / 8;
    const int lane = threadIdx.x & 31;
    if (r.slot >= 0 && lane < 2 * C) {
        const bool is_v = lane >= C;
        const int ch = is_v ? lane - C : lane;
        const uint32_t addr = (is_v ? vbase : kbase) + (ch >> 3) * tile_stride + swz(row, ch & 7);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(r.chunk.x), "r"(r.chunk.y),
                     "r"(r.chunk.z), "r"(r.chunk.w)
                     : "memory");
        if (write) {
            uint4 *dst = (is_v ? a.v_cache : a.k_cache) + r.dst + ch;
            *dst = r.chunk;
        }
        // the stage is refilled by TMA later: order these writes before that
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncwarp();
}

// Outputs of empty sequences are zero (in every layer); also flag out-of-range
// lengths. Run by CTA 0.
template <int D>
__device__ __forceinline__ void zero_empty_outputs(const DecodeArgs &a, int tid, int nthreads)
{
    const int row16 = a.Hq * D * (a.out_f32 ? 2 : 1);  // 16-bit words per output row
    for (int lb = tid; lb < a.L * a.B; lb += nthreads) {
        const int b = lb % a.B;
        const int c = __ldg(a.context_lens + b);
        if (lb < a.B && (c < 0 || c > a.W * kBlockTokens))
            atomicOr(a.status, KV_STATUS_BAD_CONTEXT);
        if (clamp_ctx(c, a.W) == 0) {
            uint16_t *o = a.out + static_cast<size_t>(lb) * row16;
            for (int i = 0; i < row16; ++i)
                o[i] = 0;  // +0.0 in both element types and in fp32
        }
    }
}

// Lane i (< m) reads the block id of unit cur.off + i of sequence cur.b; ids
// outside the pool are replaced by block 0 (never read out of bounds) and
// flagged: in the status word, or, for a read made before the grid dependency
// wait (the workspace is the previous kernel's until then), in *bad, for the
// caller to report after the wait.
__device__ __forceinline__ int load_block_ids(const DecodeArgs &a, const Cursor &cur, int m, int lane,
                                              int *bad = nullptr)
{
    int blk = 0;
    if (lane < m) {
        blk = __ldg(a.block_tables + static_cast<size_t>(cur.b) * a.W + cur.off + lane);
        if (blk < 0 || blk >= a.num_blocks) {
            if (bad)
                *bad = 1;
            else
                atomicOr(a.status, KV_STATUS_BAD_BLOCK_ID);
            blk = 0;
        }
    }
    return blk;
}

template <class E, int D, int PATH, int NH>
__global__ void __launch_bounds__(kThreads, kCtasPerSm)
    decode_kernel(const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
                  const DecodeArgs a)
{
    using G = Geo<D>;
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    unsigned char *base = smem_raw + (base_s - raw_s);
    uint64_t *full = reinterpret_cast<uint64_t *>(base + G::kOffBar);
    uint64_t *empty = full + G::kMaxStages;
    volatile int *misc = reinterpret_cast<volatile int *>(base + G::kOffMisc);
    float *scratch = reinterpret_cast<float *>(base + G::kOffScratch);
    uint64_t *qbar = reinterpret_cast<uint64_t *>(base + G::kOffQBar);  // [0,4): full, [4,8): empty

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int S = a.stages;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], a.hg);  // the HG warps of the consuming stream
        }
        for (int q = 0; q < 2 * kPieceQueue; ++q)
            mbar_init(qbar + q, 1);
        mbar_fence_init();
        misc[kMiscAbort] = 0;
        misc[kMiscLocB] = -1;
        misc[kMiscEndFound] = 0;
        misc[kMiscStartFound] = 0;
        misc[kMiscZero] = 0;
    }
    if (warp == kProducerWarp && lane == 0) {
        tma_prefetch_descriptor(&tmK);
        tma_prefetch_descriptor(&tmV);
    }
    __syncthreads();

    // ---- split plan (reads only tables and lengths: no wait needed yet) ----
    volatile long long *scan64 = reinterpret_cast<volatile long long *>(misc + kMiscScan64);
    const int w = a.item_cost;
    long long mine = 0;
    for (int b = tid; b < a.B; b += kThreads)
        mine += seq_scan_value(a, ctx_blocks(seq_ctx(a, b)));
    long long sum64;
    block_scan_incl64(mine, scan64, &sum64);
    // Work positions of one layer; every layer has the same (tables and lengths are shared), and
    // layer l's positions follow layer l - 1's.
    const int per_layer = static_cast<int>(sum64 >> kNonEmptyBits);
    const int nonempty = static_cast<int>(sum64 & ((1 << kNonEmptyBits) - 1));
    const int units_layer = per_layer - w * a.items_per_seq * nonempty;
    const int total = a.L * per_layer;  // the host checked that it fits
    int chunk = (total + static_cast<int>(gridDim.x) - 1) / static_cast<int>(gridDim.x);
    if (chunk < a.min_chunk)
        chunk = a.min_chunk;
    const int start = static_cast<int>(blockIdx.x) * chunk;
    const int end = min(start + chunk, total);

    if (start < total) {
        // locate the CTA's first unit and count the units in [start, end): the layer of each end
        // by division, the position within the layer by a scan over the sequences
        const int ls = start / per_layer, ss = start - ls * per_layer;
        const int le = (end - 1) / per_layer, se = end - 1 - le * per_layer;
        long long running = 0;
        for (int base_b = 0; base_b < a.B; base_b += kThreads) {
            const int b = base_b + tid;
            const int n = (b < a.B) ? ctx_blocks(seq_ctx(a, b)) : 0;
            const long long v = seq_scan_value(a, n);
            long long tot;
            const long long before = running + block_scan_incl64(v, scan64, &tot) - v;
            const int lo = static_cast<int>(before >> kNonEmptyBits);
            const int hi = lo + static_cast<int>(v >> kNonEmptyBits);
            const int units_before = lo - w * a.items_per_seq * static_cast<int>(before & ((1 << kNonEmptyBits) - 1));
            if (n > 0 && ss >= lo && ss < hi) {
                const int r = ss - lo, k = r / (n + w), rr = r - k * (n + w);
                misc[kMiscLocLayer] = ls;
                misc[kMiscLocB] = b;
                misc[kMiscLocK] = k;
                misc[kMiscLocOff] = max(0, rr - w);
                misc[kMiscLocPos] = ls * per_layer + lo + k * (n + w) + w;
                misc[kMiscStartU] = ls * units_layer + units_before + k * n + max(0, rr - w);
                misc[kMiscStartFound] = 1;
            }
            if (n > 0 && se >= lo && se < hi) {
                const int r = se - lo, k = r / (n + w), rr = r - k * (n + w);
                misc[kMiscEndU] = le * units_layer + units_before + k * n + max(0, rr - w) + (rr >= w ? 1 : 0);
                misc[kMiscEndFound] = 1;
            }
            running += tot;
            __syncthreads();
            if (misc[kMiscEndFound] && misc[kMiscStartFound])
                break;
        }
    }
    const int count = start < total ? misc[kMiscEndU] - misc[kMiscStartU] : 0;

    if (count <= 0) {
        grid_dependency_wait();
        grid_launch_dependents();
        if (blockIdx.x == 0)
            zero_empty_outputs<D>(a, tid, kThreads);
        return;
    }

    Cursor cur0;
    cur0.layer = misc[kMiscLocLayer];
    cur0.b = misc[kMiscLocB];
    cur0.ctx = seq_ctx(a, cur0.b);
    cur0.n = ctx_blocks(cur0.ctx);
    cur0.k = misc[kMiscLocK];
    cur0.off = misc[kMiscLocOff];
    cur0.pos = misc[kMiscLocPos];
    volatile int *abort_flag = misc + kMiscAbort;
    const uint32_t ring = base_s;

    if (warp == kProducerWarp) {
        // ---------------- producer: block ids -> TMA loads ----------------
        // The first batch of block ids is read before waiting on the previous
        // grid (the tables must not come from the kernel launched just before);
        // the cache is only touched after the wait.
        int bad_first = 0;
        const int m_first = min(32, min(cur0.n - cur0.off, count));
        int blk_first = load_block_ids(a, cur0, m_first, lane, &bad_first);
        const uint64_t policy = a.l2_policy == 2   ? l2_policy_evict_normal()
                                : a.l2_policy == 3 ? l2_policy_evict_last()
                                                   : l2_policy_evict_first();
        // With the caller's promise that the kernel before this one does not write the caches, the first
        // ring of tile loads goes out before the wait (lane i: unit i into stage i, their first use), so the
        // CTA's first data arrives while the previous kernel finishes. q and the new rows still wait.
        const int pre = a.early_loads ? min(S, m_first) : 0;
        const bool drop_here = misc[kMiscStartU] == 0;  // the test hook's CTA: it holds the launch's first unit
        if (lane < pre && !(lane == a.drop_unit && drop_here)) {
            const int head0 = (cur0.k / a.hchunks) * a.hg;
            mbar_arrive_expect_tx(&full[lane], a.stage_bytes);
            const uint32_t dst = ring + lane * a.stage_bytes;
#pragma unroll
            for (int t = 0; t < G::kTiles; ++t)
                tma_load_5d(dst + t * a.tile_stride, &tmK, t * 64, 0, head0, blk_first, cur0.layer, &full[lane],
                            policy);
#pragma unroll
            for (int t = 0; t < G::kTiles; ++t)
                tma_load_5d(dst + (G::kTiles + t) * a.tile_stride, &tmV, t * 64, 0, head0, blk_first, cur0.layer,
                            &full[lane], policy);
        }
        grid_dependency_wait();
        grid_launch_dependents();
        if (bad_first)
            atomicOr(a.status, KV_STATUS_BAD_BLOCK_ID);
        const int NL = a.prod_lanes;
        Cursor cur = cur0;
        int u = 0, issued = 0;  // units [0, issued) issued in order (every lane of their round got through)
        unsigned went = 0;      // if a round stopped midway: unit issued + l was issued (bit l, l < NL)
        bool stop = false, first_batch = true;
        while (u < count && !stop) {
            const int run = min(cur.n - cur.off, count - u);
            const int head0 = (cur.k / a.hchunks) * a.hg;
            for (int bi = 0; bi < run && !stop; bi += 32) {
                const int m = min(32, run - bi);
                int blk;
                if (first_batch) {
                    blk = blk_first;
                    first_batch = false;
                } else {
                    Cursor at = cur;
                    at.off = cur.off + bi;
                    blk = load_block_ids(a, at, m, lane);
                }
                for (int i0 = 0; i0 < m; i0 += NL) {
                    const int i = i0 + lane;
                    const int phys = __shfl_sync(kFull, blk, i & 31);
                    int ok = 1;
                    if (lane < NL && i < m && u + bi + i >= pre) {  // units below `pre` went out before the wait
                        const int uu = u + bi + i;
                        const int s = uu % S;
                        ok = mbar_wait_bounded(&empty[s], ((uu / S) & 1) ^ 1, abort_flag);
                        if (ok && uu == a.drop_unit && drop_here) {
                            // test hook: this stage is never filled, so its consumers' wait runs out
                        } else if (ok) {
                            mbar_arrive_expect_tx(&full[s], a.stage_bytes);
                            const uint32_t dst = ring + s * a.stage_bytes;
#pragma unroll
                            for (int t = 0; t < G::kTiles; ++t)
                                tma_load_5d(dst + t * a.tile_stride, &tmK, t * 64, 0, head0, phys, cur.layer,
                                            &full[s], policy);
#pragma unroll
                            for (int t = 0; t < G::kTiles; ++t)
                                tma_load_5d(dst + (G::kTiles + t) * a.tile_stride, &tmV, t * 64, 0, head0, phys,
                                            cur.layer, &full[s], policy);
                        } else {
                            *abort_flag = 1;
                            atomicOr(a.status, KV_STATUS_WAIT_TIMEOUT);
                        }
                    }
                    if (!__all_sync(kFull, ok)) {
                        went = __ballot_sync(kFull, ok && lane < NL && i < m);  // (units below `pre`: early)
                        stop = true;
                        break;
                    }
                    issued = u + bi + min(i0 + NL, m);
                }
            }
            u += run;
            if (u < count)
                cursor_next_item(a, cur);
        }
        // No load may land after this CTA exits: wait (bounded) for the last S units issued in order, and for
        // those issued in a round that stopped midway. A unit whose stage such a unit refilled had landed.
        if (lane < NL) {
            for (int v = max(0, issued - S); v < issued; ++v) {
                const int l = v + S - issued;  // the lane whose unit of the stopped round refilled v's stage
                if (v % NL == lane && !(l < NL && ((went >> l) & 1u)))
                    mbar_wait_bounded(&full[v % S], (v / S) & 1, misc + kMiscZero);
            }
            if ((went >> lane) & 1u)
                mbar_wait_bounded(&full[(issued + lane) % S], ((issued + lane) / S) & 1, misc + kMiscZero);
        }
        return;
    }

    if (warp == kHelperWarp) {
        // ------------- helper: count finished split pieces in -------------
        // For each split piece the consumers finished (other than their last),
        // release its partial and count it in; if that completes the item, merge
        // the item here. Waiting for the release is this warp's job, not theirs.
        grid_dependency_wait();
        grid_launch_dependents();
        if (!a.fused)
            return;
        for (int k = 0;; ++k) {
            const int q = k % kPieceQueue;
            if (!mbar_wait_bounded(qbar + q, (k / kPieceQueue) & 1, abort_flag))
                break;
            const volatile int *desc = misc + kMiscQueue + 5 * q;
            const int item = desc[0], first_cta = desc[1], last_cta = desc[2], lb = desc[3], kk = desc[4];
            if (item < 0)
                break;
            int last = 0;
            if (lane == 0) {
                last = atom_add_acq_rel_gpu(a.counters + item, 1) == last_cta - first_cta;
            }
            last = __shfl_sync(kFull, last, 0);
            if (last) {
                merge_pieces_global<E, D>(a, item, first_cta, last_cta, lb, kk, lane, 32);
                __syncwarp();
                if (lane == 0)
                    a.counters[item] = 0;
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(qbar + kPieceQueue + q);
        }
        return;
    }

    // -------------------- consumers: warps 0..7 --------------------
    const int hh = warp % a.hg;          // kv head within the group
    const int stream = warp / a.hg;      // which units: u % streams == stream
    const int NS = a.streams;
    Consumer<E, D, PATH, NH> st;
    float *q_s = scratch + hh * kGroupMax * G::kQStride;                         // CUDA-core path only
    float *p_s = scratch + kMaxHG * kGroupMax * G::kQStride + warp * 16 * kGroupMax;
    grid_dependency_wait();
    grid_launch_dependents();
    // q, like the new token rows, may come from the previous kernel: load after the wait
    st.prefetch_q(a, item_out(a, cur0, hh));
    // the new token rows (fused append) are loaded after the wait: the caller may
    // have produced them in the previous kernel
    AppendRow ar_next = load_append_row<D>(a, cur0, (cur0.k / a.hchunks) * a.hg + hh,
                                           hh == 0 && (cur0.k % a.hchunks) == 0);
    if (blockIdx.x == 0)
        zero_empty_outputs<D>(a, tid, kConsumerThreads);
    Cursor cur = cur0;
    int u = 0;
    int pushed = 0;  // split pieces handed to the helper (thread 0's count)
    while (u < count) {
        const int run = min(cur.n - cur.off, count - u);
        const int item = item_index(a, cur);
        const int hg = cur.k / a.hchunks, hc = cur.k - hg * a.hchunks;
        const ItemOut o = item_out(a, cur, hh);
        const int first_cta = cur.pos / chunk;
        const int last_cta = (cur.pos + cur.n - 1) / chunk;
        const bool single = first_cta == last_cta;
        // Pieces of this item already finished elsewhere, read by the first lane of
        // a stream that does not take the item's last unit (the checker) when it
        // starts its own last unit, and judged when it has finished it: its wait
        // for the count and the acquire fence overlap the last unit's work.
        const int checker_stream = ((u + run - 1) % NS + 1) % NS;
        const bool checker = stream == checker_stream && hh == 0 && lane == 0;
        int seen = -1;

        if (PATH == kPathSimt) {
            // this item's query rows as fp32 in shared memory (heads >= gc are zero)
            const int per = kGroupMax * D;
            for (int idx = tid; idx < a.hg * per; idx += kConsumerThreads) {
                const int h2 = idx / per;
                const int rem = idx - h2 * per;
                const int n = rem / D, d = rem - n * D;
                const int h = (hg * a.hg + h2) * a.group + hc * kGroupMax + n;
                const float v =
                    (n < o.gc) ? E::to_f32(a.q[(static_cast<size_t>(o.lb) * a.Hq + h) * D + d]) : 0.f;
                scratch[(h2 * kGroupMax + n) * G::kQStride + d + ((d >= D / 2) ? 4 : 0)] = v;
            }
            named_barrier(kBarConsumers, kConsumerThreads);
        }
        st.begin_item(a, o, q_s);
        const AppendRow ar = ar_next;
        const int j_head = hg * a.hg + hh;
        if (u + run < count) {
            Cursor next = cur;
            cursor_next_item(a, next);
            st.prefetch_q(a, item_out(a, next, hh));
            ar_next = load_append_row<D>(a, next, (next.k / a.hchunks) * a.hg + hh,
                                         hh == 0 && (next.k % a.hchunks) == 0);
        }
        // this stream's units of the item: u + i, u + i + NS, ...; their stage and phase are stepped rather than
        // divided out per unit (S is a multiple of NS), which took the 0.5B per-layer step from 4.18-4.19 to
        // 4.36-4.37 TB/s on one box: the consumers' path between two units is part of what paces D = 64
        int i = ((stream - u) % NS + NS) % NS;
        int s = (u + i) % S, ph = ((u + i) / S) & 1;
        for (; i < run; i += NS) {
            if (!mbar_wait_bounded(&full[s], ph, abort_flag)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    atomicOr(a.status, KV_STATUS_WAIT_TIMEOUT);
                }
                break;
            }
            if (checker && !single && a.fused && i + NS >= run)
                seen = ld_relaxed_gpu(a.counters + item);
            const uint32_t kb = ring + s * a.stage_bytes + hh * kHeadTileBytes;
            const int valid = min(kBlockTokens, cur.ctx - (cur.off + i) * kBlockTokens);
            if (cur.off + i == cur.n - 1)  // the block holding this step's token
                apply_append_row<D>(a, ar, j_head, valid - 1, kb, kb + G::kTiles * a.tile_stride, a.tile_stride,
                                    hc == 0);
            st.unit(kb, kb + G::kTiles * a.tile_stride, a.tile_stride, valid, a.scale_log2, q_s, p_s);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[s]);
            s += NS;
            if (s >= S) {
                s -= S;
                ph ^= 1;
            }
        }
        if (checker) {
            bool solo_now = false;
            if (!single && a.fused) {
                if (seen < 0)  // the checker's stream had no unit of this item
                    seen = ld_relaxed_gpu(a.counters + item);
                solo_now = seen == last_cta - first_cta;
                if (solo_now)
                    fence_acquire_gpu();  // the other pieces' partials, before anyone reads them
            }
            misc[kMiscSolo] = solo_now ? 1 : 0;
        }
        st.finish();
        const bool final_piece = u + run == count;

        // ---- merge the streams pairwise: stream s + step hands over to stream s ----
        if (PATH == kPathSimt || NS == 1)
            named_barrier(kBarConsumers, kConsumerThreads);  // the scratch also holds q_s / p_s
        for (int step = 1; step < NS; step <<= 1) {
            const bool giver = (stream % (2 * step)) == step;
            const bool taker = (stream % (2 * step)) == 0 && stream + step < NS;
            const int slot_giver = (stream / (2 * step)) * a.hg + hh;
            const int slot_taker = ((stream + step) / (2 * step)) * a.hg + hh;
            if (giver)
                st.save(scratch + slot_giver * Consumer<E, D, PATH, NH>::kRegs * 32);
            named_barrier(kBarConsumers, kConsumerThreads);
            if (taker)
                st.merge(scratch + slot_taker * Consumer<E, D, PATH, NH>::kRegs * 32);
            named_barrier(kBarConsumers, kConsumerThreads);
        }

        // Split items: if every other piece was already done when this one started,
        // this CTA merges them now (no partial, no counter traffic). Otherwise it
        // stores its partial and counts itself in; the CTA that completes the count
        // merges from global memory -- checked at that CTA's next epilogue.
        const bool solo = misc[kMiscSolo] != 0;
        float *own_acc = scratch;                                   // the solo merge's copy of this piece
        float *own_ml = scratch + kMaxHG * kGroupMax * D;
        if (stream == 0) {
            if (single) {
                st.store_final(a, o);
            } else if (solo) {
                st.store_state(o, own_acc, own_ml);
            } else {
                const size_t slot0 = o.slot * (kMaxHG * kGroupMax);
                st.store_state(o, a.part_acc + slot0 * D, a.part_ml + slot0 * 2);
            }
        }
        if (!single && solo) {
            // every other piece is done: merge them with this one (read from shared memory)
            named_barrier(kBarConsumers, kConsumerThreads);
            merge_pieces_global<E, D>(a, item, first_cta, last_cta, o.lb, cur.k, tid, kConsumerThreads,
                                      static_cast<int>(blockIdx.x), own_acc, own_ml);
            if (tid == 0)
                a.counters[item] = 0;
        }
        named_barrier(kBarConsumers, kConsumerThreads);  // this piece's partial is written; the scratch is free
        if (!single && a.fused && !solo) {
            if (!final_piece) {
                // hand the count to the helper warp and go on streaming
                if (tid == 0) {
                    const int q = pushed % kPieceQueue;
                    if (mbar_wait_bounded(qbar + kPieceQueue + q, ((pushed / kPieceQueue) & 1) ^ 1, abort_flag)) {
                        volatile int *desc = misc + kMiscQueue + 5 * q;
                        desc[0] = item;
                        desc[1] = first_cta;
                        desc[2] = last_cta;
                        desc[3] = o.lb;
                        desc[4] = cur.k;
                        mbar_arrive(qbar + q);
                        ++pushed;
                    } else {
                        *abort_flag = 1;
                        atomicOr(a.status, KV_STATUS_WAIT_TIMEOUT);
                    }
                }
            } else {
                // the CTA's last piece: count it in and merge here if it completed the item
                if (tid == 0) {
                    const bool last = atom_add_acq_rel_gpu(a.counters + item, 1) == last_cta - first_cta;
                    misc[kMiscLast] = last ? 1 : 0;
                }
                named_barrier(kBarConsumers, kConsumerThreads);
                if (misc[kMiscLast]) {
                    merge_pieces_global<E, D>(a, item, first_cta, last_cta, o.lb, cur.k, tid, kConsumerThreads);
                    if (tid == 0)
                        a.counters[item] = 0;
                }
            }
        }
        u += run;
        if (u < count)
            cursor_next_item(a, cur);
    }
    // tell the helper there is nothing more
    if (tid == 0 && a.fused) {
        const int q = pushed % kPieceQueue;
        if (mbar_wait_bounded(qbar + kPieceQueue + q, ((pushed / kPieceQueue) & 1) ^ 1, abort_flag)) {
            misc[kMiscQueue + 5 * q] = -1;
            mbar_arrive(qbar + q);
        } else {
            *abort_flag = 1;
            atomicOr(a.status, KV_STATUS_WAIT_TIMEOUT);
        }
    }
}

// Separate split-K combine: one CTA per work item.
template <class E, int D>
__global__ void __launch_bounds__(128) combine_kernel(const DecodeArgs a, int grid_ctas)
{
    __shared__ int red[2][4];
    grid_dependency_wait();
    grid_launch_dependents();
    const int item = blockIdx.x;
    const int lb = item / a.items_per_seq, k = item - lb * a.items_per_seq;
    const int layer = lb / a.B, b = lb - layer * a.B;
    // work positions, as the decode kernel counts them
    int pre = 0, tot = 0;
    for (int bb = threadIdx.x; bb < a.B; bb += 128) {
        const int n = ctx_blocks(seq_ctx(a, bb));
        const int wpos = n > 0 ? a.items_per_seq * (n + a.item_cost) : 0;
        tot += wpos;
        pre += (bb < b) ? wpos : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        tot += __shfl_xor_sync(kFull, tot, o);
        pre += __shfl_xor_sync(kFull, pre, o);
    }
    if ((threadIdx.x & 31) == 0) {
        red[0][threadIdx.x >> 5] = tot;
        red[1][threadIdx.x >> 5] = pre;
    }
    __syncthreads();
    tot = red[0][0] + red[0][1] + red[0][2] + red[0][3];
    pre = red[1][0] + red[1][1] + red[1][2] + red[1][3];
    const int n = ctx_blocks(seq_ctx(a, b));
    if (n == 0)
        return;
    const int total = a.L * tot;  // tot: positions of one layer
    int chunk = (total + grid_ctas - 1) / grid_ctas;
    if (chunk < a.min_chunk)
        chunk = a.min_chunk;
    const int item_pos = layer * tot + pre + k * (n + a.item_cost) + a.item_cost;  // its first unit
    const int first_cta = item_pos / chunk, last_cta = (item_pos + n - 1) / chunk;
    if (first_cta == last_cta)
        return;
    merge_pieces_global<E, D>(a, item, first_cta, last_cta, lb, k, threadIdx.x, 128);
}

}  // namespace pkv

// ===========================================================================
// Host side
// ===========================================================================
namespace {

using namespace pkv;

std::atomic<int> g_opt_compute{0};
std::atomic<int> g_opt_combine{0};
std::atomic<int> g_opt_grid{0};
std::atomic<int> g_opt_min_chunk{0};
std::atomic<int> g_opt_prod_lanes{0};
std::atomic<int> g_opt_head_group{0};
std::atomic<int> g_opt_item_cost{0};
std::atomic<int> g_opt_prefill_path{0};
std::atomic<int> g_opt_drop_load{0};
std::atomic<int> g_opt_slow_softmax{0};
std::atomic<int> g_opt_out_f32{0};
std::atomic<int> g_opt_l2_policy{0};
std::atomic<int> g_opt_early_loads{0};
constexpr int kDefaultMinChunk = 4;

// Work positions charged per work item (its fixed cost, in units of one work
// unit's streaming time): the KV_OPT_ITEM_COST setting, else a measured default.
// A CTA that crosses an item boundary stops both streams to merge and hand off
// a piece (~3 us in a timestamp trace of the 0.5B layer); a D = 64 unit streams
// in ~0.3 us, a D = 128 unit in ~0.6 us.
int item_cost(int D)
{
    const int v = g_opt_item_cost.load();
    if (v < 0)
        return 0;
    if (v > 0)
        return v;
    return D == 64 ? 10 : 6;
}

constexpr int kMaxDevices = 64;

int device_sm_count(int dev)
{
    static std::atomic<int> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices)
        return 0;
    int v = cache[dev].load();
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return 0;
        cache[dev].store(v);
    }
    return v;
}

// kv heads per work unit: 4 when Hkv is a multiple of 4, else 2 or 1 (or the
// KV_OPT_HEAD_GROUP setting when it divides Hkv)
int heads_per_unit(int Hkv)
{
    const int want = g_opt_head_group.load();
    if (want > 0 && Hkv % want == 0)
        return want;
    return Hkv % 4 == 0 ? 4 : (Hkv % 2 == 0 ? 2 : 1);
}

struct Layout {
    int items = 0, slots = 0, max_grid = 0;
    size_t off_counters = 0, off_ml = 0, off_acc = 0, bytes = 0;
};

size_t round256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// Workspace of a launch over `layers` layers of B sequences on a device with
// `sms` SMs: the status word, one counter per work item, and per split-K piece
// slot (m, l) and the accumulator.
bool make_layout(int B, int Hq, int Hkv, int D, int layers, int sms, Layout *lay)
{
    if (B < 0 || layers < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || (D != 64 && D != 128) || sms < 1)
        return false;
    const int group = Hq / Hkv;
    const long long hchunks = (group + kGroupMax - 1) / kGroupMax;
    const long long items =
        static_cast<long long>(layers) * B * (Hkv / heads_per_unit(Hkv)) * hchunks;
    if (items > (1ll << 30))
        return false;
    lay->items = static_cast<int>(items);
    lay->max_grid = kCtasPerSm * sms;
    lay->slots = lay->max_grid + lay->items;
    lay->off_counters = kStatusBytes;
    lay->off_ml = lay->off_counters + round256(static_cast<size_t>(lay->items) * 4);
    lay->off_acc = lay->off_ml + round256(static_cast<size_t>(lay->slots) * kMaxHG * kGroupMax * 2 * 4);
    lay->bytes = lay->off_acc + round256(static_cast<size_t>(lay->slots) * kMaxHG * kGroupMax * D * 4);
    return true;
}

using DecodeFn = void (*)(const CUtensorMap, const CUtensorMap, const DecodeArgs);

template <class E>
DecodeFn pick_kernel_for(int D, int path, int nh, int *smem)
{
#define PKV_CASE(DD, PP, NN)                          \
    if (D == DD && path == PP && nh == NN) {          \
        *smem = Geo<DD>::kSmemBytes;                  \
        return decode_kernel<E, DD, PP, NN>;          \
    }
    PKV_CASE(64, kPathMma, 8)
    PKV_CASE(128, kPathMma, 8)
    PKV_CASE(64, kPathSimt, 1)
    PKV_CASE(64, kPathSimt, 2)
    PKV_CASE(64, kPathSimt, 4)
    PKV_CASE(64, kPathSimt, 8)
    PKV_CASE(128, kPathSimt, 1)
    PKV_CASE(128, kPathSimt, 2)
    PKV_CASE(128, kPathSimt, 4)
    PKV_CASE(128, kPathSimt, 8)
#undef PKV_CASE
    return nullptr;
}

DecodeFn pick_kernel(int dtype, int D, int path, int nh, int *smem)
{
    return dtype == KV_DTYPE_FP16 ? pick_kernel_for<ElemF16>(D, path, nh, smem)
                                  : pick_kernel_for<ElemBf16>(D, path, nh, smem);
}

// Per (kernel, device): dynamic shared memory opted in, and resident CTAs per SM.
int prepare_kernel(DecodeFn fn, int smem, int dev)
{
    struct Entry {
        const void *fn;
        int dev;
        int occ;
    };
    static std::mutex mu;
    static Entry table[64];
    static int used = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (table[i].fn == reinterpret_cast<const void *>(fn) && table[i].dev == dev)
            return table[i].occ;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return 0;
    int occ = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, fn, kThreads, smem) != cudaSuccess)
        return 0;
    if (used < 64)
        table[used++] = Entry{reinterpret_cast<const void *>(fn), dev, occ};
    return occ;
}

bool misaligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; }

// A checked decode launch: everything it needs, built on the host before
// anything is enqueued. grid == 0 means there is nothing to launch (B == 0).
struct DecodePlan {
    DecodeFn fn = nullptr;
    int smem = 0, grid = 0, dtype = 0, D = 0;
    Layout lay;
    CUtensorMap tmK, tmV;
    DecodeArgs a;
};

// Validate a decode over `layers` layers (k_new == nullptr: no append) and fill
// *p. Enqueues nothing; KV_ERR_ARG / KV_ERR_CUDA as the entry points document.
// cache_layer_stride is in elements (ignored when layers == 1).
kv_status plan_decode(DecodePlan *p, void *out, const void *q, const void *k_new, const void *v_new,
                      const void *k_cache, const void *v_cache, size_t cache_layer_stride, int layers,
                      const int64_t *slot_mapping, const int32_t *block_tables, int max_blocks_per_seq,
                      const int32_t *context_lens, int B, int num_blocks, int Hq, int Hkv, int D, float scale,
                      int dtype, void *workspace, size_t workspace_bytes)
{
    p->grid = 0;
    if ((dtype != KV_DTYPE_BF16 && dtype != KV_DTYPE_FP16) || B < 0 || layers < 1 || max_blocks_per_seq < 1 ||
        num_blocks < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || (D != 64 && D != 128))
        return KV_ERR_ARG;
    if (B == 0)
        return KV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !workspace)
        return KV_ERR_ARG;
    if (misaligned(out, 16) || misaligned(q, 16) || misaligned(k_cache, 16) || misaligned(v_cache, 16) ||
        misaligned(block_tables, 4) || misaligned(context_lens, 4) || misaligned(workspace, 256))
        return KV_ERR_ARG;
    const size_t layer_elems = static_cast<size_t>(num_blocks) * kBlockTokens * Hkv * D;
    if (layers == 1)
        cache_layer_stride = layer_elems;  // the map's layer dimension has one entry
    else if (cache_layer_stride < layer_elems || cache_layer_stride % 8 != 0 ||
             cache_layer_stride > (static_cast<size_t>(1) << 38))
        return KV_ERR_ARG;  // overlapping layers, a stride that is not a multiple of 16 bytes, or too large
    const int group = Hq / Hkv;
    const int hg = heads_per_unit(Hkv);
    const int hchunks = (group + kGroupMax - 1) / kGroupMax;
    const int cost = item_cost(D);
    if (static_cast<long long>(layers) * B * (max_blocks_per_seq + cost) * (Hkv / hg) * hchunks >= (1ll << 31) ||
        B >= (1 << 24))
        return KV_ERR_ARG;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return KV_ERR_CUDA;
    const int sms = device_sm_count(dev);
    if (!make_layout(B, Hq, Hkv, D, layers, sms, &p->lay))
        return KV_ERR_ARG;
    if (workspace_bytes < p->lay.bytes)
        return KV_ERR_ARG;

    int path = g_opt_compute.load();
    if (path == 0)
        path = kPathMma;
    int nh = kGroupMax;
    if (path == kPathSimt) {
        const int gmin = group < kGroupMax ? group : kGroupMax;
        nh = gmin <= 1 ? 1 : gmin <= 2 ? 2 : gmin <= 4 ? 4 : 8;
    }
    p->fn = pick_kernel(dtype, D, path, nh, &p->smem);
    if (!p->fn)
        return KV_ERR_ARG;
    const int occ = prepare_kernel(p->fn, p->smem, dev);
    if (occ < 1)
        return KV_ERR_CUDA;
    int grid = (occ < kCtasPerSm ? occ : kCtasPerSm) * sms;
    const int want = g_opt_grid.load();
    if (want > 0)
        grid = want < p->lay.max_grid ? want : p->lay.max_grid;

    // ring geometry: stages a multiple of the consumer streams and of the producer lanes
    const int tiles = D / 64;
    const int streams = kConsumerWarps / hg;
    int lanes = g_opt_prod_lanes.load();
    if (lanes <= 0)
        lanes = hg >= 2 ? 2 : 4;  // one lane cannot issue a D = 64 unit's two boxes as fast as 148 SMs drain them
    const int stage_bytes = 2 * tiles * hg * kHeadTileBytes;
    const int unit_of = streams > lanes ? streams : lanes;
    const int ring = D == 64 ? Geo<64>::kRingBytes : Geo<128>::kRingBytes;
    const int max_stages = D == 64 ? Geo<64>::kMaxStages : Geo<128>::kMaxStages;
    int stages = (ring / stage_bytes) / unit_of * unit_of;
    if (stages > max_stages)
        stages = max_stages / unit_of * unit_of;
    if (stages < unit_of)
        return KV_ERR_ARG;

    const unsigned long long stride_bytes = static_cast<unsigned long long>(cache_layer_stride) * 2;
    if (!pkv_host::make_layered_cache_map(&p->tmK, k_cache, num_blocks, Hkv, D, hg, dtype, layers, stride_bytes) ||
        !pkv_host::make_layered_cache_map(&p->tmV, v_cache, num_blocks, Hkv, D, hg, dtype, layers, stride_bytes))
        return KV_ERR_CUDA;

    unsigned char *ws = static_cast<unsigned char *>(workspace);
    DecodeArgs &a = p->a;
    a.out = static_cast<uint16_t *>(out);
    a.q = static_cast<const uint16_t *>(q);
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.part_acc = reinterpret_cast<float *>(ws + p->lay.off_acc);
    a.part_ml = reinterpret_cast<float *>(ws + p->lay.off_ml);
    a.counters = reinterpret_cast<int32_t *>(ws + p->lay.off_counters);
    a.status = reinterpret_cast<int32_t *>(ws);
    a.B = B;
    a.W = max_blocks_per_seq;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.group = group;
    a.num_blocks = num_blocks;
    a.L = layers;
    a.out_f32 = g_opt_out_f32.load();
    a.hg = hg;
    a.streams = streams;
    a.hchunks = hchunks;
    a.items_per_seq = (Hkv / hg) * hchunks;
    a.stages = stages;
    a.stage_bytes = stage_bytes;
    a.tile_stride = hg * kHeadTileBytes;
    a.prod_lanes = lanes;
    const int mc = g_opt_min_chunk.load();
    a.min_chunk = mc > 0 ? mc : kDefaultMinChunk;
    a.item_cost = cost;
    a.drop_unit = g_opt_drop_load.load() - 1;
    // Auto, as measured on this GPU (one box, both priorities twice per workload): evict-first for a single
    // layer and for multi-layer launches at D = 64 (0.5B step 6.39 -> 6.74 TB/s against evict-normal);
    // evict-normal for multi-layer launches at D = 128 (LLaMA shapes +2 %, and +11 % on the shared-prefix
    // mix, whose prefix blocks are re-read far apart while every layer is in flight).
    a.l2_policy = g_opt_l2_policy.load() != 0 ? g_opt_l2_policy.load() : ((layers > 1 && D == 128) ? 2 : 1);
    a.early_loads = g_opt_early_loads.load();
    a.fused = g_opt_combine.load() == 0 ? 1 : 0;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.append = k_new != nullptr ? 1 : 0;
    a.k_new = static_cast<const uint4 *>(k_new);
    a.v_new = static_cast<const uint4 *>(v_new);
    a.k_cache = static_cast<uint4 *>(const_cast<void *>(k_cache));
    a.v_cache = static_cast<uint4 *>(const_cast<void *>(v_cache));
    a.cache_layer_chunks = cache_layer_stride / 8;
    a.slots = slot_mapping;
    p->grid = grid;
    p->dtype = dtype;
    p->D = D;
    return KV_OK;
}

// Enqueue a planned decode (and the separate combine kernel when that mode is set).
kv_status launch_decode(const DecodePlan &p, kv_stream_t stream)
{
    if (p.grid == 0)
        return KV_OK;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = p.smem;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, p.fn, p.tmK, p.tmV, p.a) != cudaSuccess)
        return KV_ERR_CUDA;

    if (!p.a.fused) {
        cudaLaunchConfig_t c2 = {};
        c2.gridDim = dim3(p.lay.items);
        c2.blockDim = dim3(128);
        c2.dynamicSmemBytes = 0;
        c2.stream = st;
        c2.attrs = attr;
        c2.numAttrs = 1;
        cudaError_t e;
        if (p.dtype == KV_DTYPE_FP16)
            e = (p.D == 64) ? cudaLaunchKernelEx(&c2, combine_kernel<ElemF16, 64>, p.a, p.grid)
                            : cudaLaunchKernelEx(&c2, combine_kernel<ElemF16, 128>, p.a, p.grid);
        else
            e = (p.D == 64) ? cudaLaunchKernelEx(&c2, combine_kernel<ElemBf16, 64>, p.a, p.grid)
                            : cudaLaunchKernelEx(&c2, combine_kernel<ElemBf16, 128>, p.a, p.grid);
        if (e != cudaSuccess)
            return KV_ERR_CUDA;
    }
    return KV_OK;
}

}  // namespace

extern "C" size_t paged_attention_workspace_size(int B, int Hq, int Hkv, int D)
{
    return paged_attention_workspace_size_layers(B, Hq, Hkv, D, 1);
}

extern "C" size_t paged_attention_workspace_size_layers(int B, int Hq, int Hkv, int D, int num_layers)
{
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return 0;
    Layout lay;
    if (!make_layout(B, Hq, Hkv, D, num_layers, device_sm_count(dev), &lay))
        return 0;
    return lay.bytes;
}

extern "C" kv_status paged_attention_workspace_init(void *workspace, size_t workspace_bytes, kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("paged_attention_workspace_init");
    if (!workspace || workspace_bytes == 0)
        return KV_ERR_ARG;
    return cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream)) == cudaSuccess
               ? KV_OK
               : KV_ERR_CUDA;
}

extern "C" kv_status paged_attention_decode(void *out, const void *q, const void *k_cache, const void *v_cache,
                                            const int32_t *block_tables, int max_blocks_per_seq,
                                            const int32_t *context_lens, int B, int num_blocks, int Hq, int Hkv,
                                            int D, float scale, int dtype, void *workspace,
                                            size_t workspace_bytes, kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("paged_attention_decode");
    DecodePlan p;
    const kv_status r = plan_decode(&p, out, q, nullptr, nullptr, k_cache, v_cache, 0, 1, nullptr, block_tables,
                                    max_blocks_per_seq, context_lens, B, num_blocks, Hq, Hkv, D, scale, dtype,
                                    workspace, workspace_bytes);
    return r != KV_OK ? r : launch_decode(p, stream);
}

extern "C" kv_status paged_attention_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                                                   void *k_cache, void *v_cache, const int64_t *slot_mapping,
                                                   const int32_t *block_tables, int max_blocks_per_seq,
                                                   const int32_t *context_lens, int B, int num_blocks, int Hq,
                                                   int Hkv, int D, float scale, int dtype, void *workspace,
                                                   size_t workspace_bytes, kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("paged_attention_decode_append");
    if (!k_new || !v_new || !slot_mapping || misaligned(k_new, 16) || misaligned(v_new, 16) ||
        misaligned(slot_mapping, 8))
        return KV_ERR_ARG;
    DecodePlan p;
    const kv_status r = plan_decode(&p, out, q, k_new, v_new, k_cache, v_cache, 0, 1, slot_mapping, block_tables,
                                    max_blocks_per_seq, context_lens, B, num_blocks, Hq, Hkv, D, scale, dtype,
                                    workspace, workspace_bytes);
    return r != KV_OK ? r : launch_decode(p, stream);
}

extern "C" kv_status paged_attention_decode_layers(void *out, const void *q, const void *k_new, const void *v_new,
                                                   void *k_cache, void *v_cache, size_t cache_layer_stride,
                                                   int num_layers, const int64_t *slot_mapping,
                                                   const int32_t *block_tables, int max_blocks_per_seq,
                                                   const int32_t *context_lens, int B, int num_blocks, int Hq,
                                                   int Hkv, int D, float scale, int dtype, void *workspace,
                                                   size_t workspace_bytes, kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("paged_attention_decode_layers");
    const bool append = k_new != nullptr;
    if (append != (v_new != nullptr) || append != (slot_mapping != nullptr))
        return KV_ERR_ARG;  // the new rows and their slots come together, or not at all
    if (append && (misaligned(k_new, 16) || misaligned(v_new, 16) || misaligned(slot_mapping, 8)))
        return KV_ERR_ARG;
    DecodePlan p;
    const kv_status r = plan_decode(&p, out, q, k_new, v_new, k_cache, v_cache, cache_layer_stride, num_layers,
                                    slot_mapping, block_tables, max_blocks_per_seq, context_lens, B, num_blocks, Hq,
                                    Hkv, D, scale, dtype, workspace, workspace_bytes);
    return r != KV_OK ? r : launch_decode(p, stream);
}

// ---------------------------------------------------------------------------
// Decode without caller-provided workspace.
//
// For callers that cannot allocate device memory themselves: a plugin running
// inside a host program that owns every device allocation, or a code path
// where the implicit device synchronisation of cudaMalloc is not allowed. The
// split-K scratch lives in one fixed array in this library's device image
// instead, held by every GPU that loads the library until the process exits.
// ---------------------------------------------------------------------------
namespace {
constexpr size_t kNoAllocScratchBytes = KV_NOALLOC_SCRATCH_BYTES;

typedef CUresult (*CtxGetCurrentFn)(CUcontext *);

CUcontext current_context()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(p);
    });
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS)
        return nullptr;
    return c;
}
}  // namespace
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

namespace {
// The array's device address on device `dev` (current). In host code the
// array's name is a host-side stand-in, not a device address, so it is looked
// up with cudaGetSymbolAddress: once per device, and again if the device's
// current context changed since (a context created anew loads the module anew).
void *noalloc_scratch(int dev)
{
    struct Entry {
        CUcontext ctx;
        void *ptr;
    };
    static std::mutex mu;
    static Entry cache[kMaxDevices];
    std::lock_guard<std::mutex> lock(mu);
    CUcontext ctx = current_context();
    if (ctx != nullptr && cache[dev].ctx == ctx && cache[dev].ptr != nullptr)
        return cache[dev].ptr;
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p)
        return nullptr;
    cache[dev].ctx = current_context();  // the runtime has made the device's context current by now
    cache[dev].ptr = p;
    return p;
}
}  // namespace

extern "C" kv_status paged_attention_decode_noalloc(void *out, const void *q, const void *k_cache,
                                                    const void *v_cache, const int32_t *block_tables,
                                                    int max_blocks_per_seq, const int32_t *context_lens, int B,
                                                    int num_blocks, int Hq, int Hkv, int D, float scale, int dtype,
                                                    kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("paged_attention_decode_noalloc");
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return KV_ERR_CUDA;
    void *ws = noalloc_scratch(dev);
    if (!ws)
        return KV_ERR_CUDA;
    // every check first (a scratch larger than the array is KV_ERR_ARG): a rejected call touches nothing
    DecodePlan p;
    const kv_status r = plan_decode(&p, out, q, nullptr, nullptr, k_cache, v_cache, 0, 1, nullptr, block_tables,
                                    max_blocks_per_seq, context_lens, B, num_blocks, Hq, Hkv, D, scale, dtype, ws,
                                    kNoAllocScratchBytes);
    if (r != KV_OK || p.grid == 0)
        return r;
    // The array keeps the previous call's contents: the status word and the
    // per-item counters must start at zero.
    if (cudaMemsetAsync(ws, 0, p.lay.off_ml, reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
        return KV_ERR_CUDA;
    return launch_decode(p, stream);
}

extern "C" kv_status paged_attention_read_status(const void *workspace, int32_t *status_out, int clear,
                                                 kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("paged_attention_read_status");
    if (!workspace || !status_out)
        return KV_ERR_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(st) != cudaSuccess)
        return KV_ERR_CUDA;
    if (cudaMemcpy(status_out, workspace, sizeof(int32_t), cudaMemcpyDeviceToHost) != cudaSuccess)
        return KV_ERR_CUDA;
    if (clear && cudaMemset(const_cast<void *>(workspace), 0, sizeof(int32_t)) != cudaSuccess)
        return KV_ERR_CUDA;
    return KV_OK;
}

extern "C" kv_status kv_decode_set_option(int key, int value)
{
    switch (key) {
    case KV_OPT_COMPUTE:
        if (value < 0 || value > 2)
            return KV_ERR_ARG;
        g_opt_compute.store(value);
        return KV_OK;
    case KV_OPT_COMBINE:
        if (value < 0 || value > 1)
            return KV_ERR_ARG;
        g_opt_combine.store(value);
        return KV_OK;
    case KV_OPT_GRID:
        if (value < 0)
            return KV_ERR_ARG;
        g_opt_grid.store(value);
        return KV_OK;
    case KV_OPT_MIN_CHUNK:
        if (value < 0)
            return KV_ERR_ARG;
        g_opt_min_chunk.store(value);
        return KV_OK;
    case KV_OPT_PRODUCER_LANES:
        if (value < 0 || value > 8 || (value & (value - 1)) != 0)
            return KV_ERR_ARG;
        g_opt_prod_lanes.store(value);
        return KV_OK;
    case KV_OPT_HEAD_GROUP:
        if (value != 0 && value != 1 && value != 2 && value != 4)
            return KV_ERR_ARG;
        g_opt_head_group.store(value);
        return KV_OK;
    case KV_OPT_ITEM_COST:
        if (value < -1 || value > 64)
            return KV_ERR_ARG;
        g_opt_item_cost.store(value);
        return KV_OK;
    case KV_OPT_PREFILL_PATH:
        if (value < 0 || value > 3)
            return KV_ERR_ARG;
        g_opt_prefill_path.store(value);
        return KV_OK;
    case KV_OPT_TEST_DROP_LOAD:
        if (value < 0)
            return KV_ERR_ARG;
        g_opt_drop_load.store(value);
        return KV_OK;
    case KV_OPT_TEST_SLOW_SOFTMAX:
        if (value < 0 || value > 1)
            return KV_ERR_ARG;
        g_opt_slow_softmax.store(value);
        return KV_OK;
    case KV_OPT_OUT_F32:
        if (value < 0 || value > 1)
            return KV_ERR_ARG;
        g_opt_out_f32.store(value);
        return KV_OK;
    case KV_OPT_L2_POLICY:
        if (value < 0 || value > 3)
            return KV_ERR_ARG;
        g_opt_l2_policy.store(value);
        return KV_OK;
    case KV_OPT_EARLY_LOADS:
        if (value < 0 || value > 1)
            return KV_ERR_ARG;
        g_opt_early_loads.store(value);
        return KV_OK;
    default:
        return KV_ERR_ARG;
    }
}

extern "C" int kv_decode_get_option(int key)
{
    switch (key) {
    case KV_OPT_COMPUTE:
        return g_opt_compute.load();
    case KV_OPT_COMBINE:
        return g_opt_combine.load();
    case KV_OPT_GRID:
        return g_opt_grid.load();
    case KV_OPT_MIN_CHUNK:
        return g_opt_min_chunk.load();
    case KV_OPT_PRODUCER_LANES:
        return g_opt_prod_lanes.load();
    case KV_OPT_HEAD_GROUP:
        return g_opt_head_group.load();
    case KV_OPT_ITEM_COST:
        return g_opt_item_cost.load();
    case KV_OPT_PREFILL_PATH:
        return g_opt_prefill_path.load();
    case KV_OPT_TEST_DROP_LOAD:
        return g_opt_drop_load.load();
    case KV_OPT_TEST_SLOW_SOFTMAX:
        return g_opt_slow_softmax.load();
    case KV_OPT_OUT_F32:
        return g_opt_out_f32.load();
    case KV_OPT_L2_POLICY:
        return g_opt_l2_policy.load();
    case KV_OPT_EARLY_LOADS:
        return g_opt_early_loads.load();
    default:
        return -1;
    }
}

// The prefill path switch and test hook (read by prefill.cu).
int pkv_prefill_path() { return g_opt_prefill_path.load(); }
int pkv_prefill_slow_softmax() { return g_opt_slow_softmax.load(); }
int pkv_out_f32() { return g_opt_out_f32.load(); }

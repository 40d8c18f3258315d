// paged_attention_prefill: chunked-prefill attention over a paged KV cache, for
// sm_100a.
//
// What is computed ("Module 23: Serving", section 23.2, Prefill and Decode;
// "Designing an LLM serving system", section "Scheduling: when prefill meets
// decode": a long prompt is split into chunks processed between decode steps):
// sequence b has c_b tokens in the cache, the last n_b of which are this
// chunk's (already appended). Chunk token i sits at position p = c_b - n_b + i
// and attends causally to cache positions 0..p, with query head h reading kv
// head h / (Hq / Hkv):
//     out[i][h] = sum_{t <= p} softmax_t(scale * <q[i][h], K_t>) V_t.
//
// Work decomposition. The query rows of one (sequence, kv head) are the chunk's
// tokens times the group's query heads, token-major (the group's heads share
// every K/V tile); a CTA takes a run of them and reads the sequence's KV blocks
// up to the last position among its rows. Three kernels compute it, chosen by
// KV_OPT_PREFILL_PATH: two tiles of 128 rows per CTA on tcgen05 (the default,
// last in this file), one tile of 128 rows per CTA on tcgen05 (path 1), and
// the mma.sync kernel below (path 2), kept as the comparison.
//
// mma.sync kernel. 64 rows per CTA (4 warps x 16 rows); CTAs with later rows
// (more KV) are launched first. Warp 4 is the producer: it reads block ids and
// issues TMA loads of 4 KV blocks (64 tokens) per stage into a ring of 3
// stages, guarded by mbarriers with bounded waits. Warps 0-3 compute with
// mma.sync.m16n8k16 (16-bit inputs, fp32 accumulate): per stage
// S[16 rows x 64 tokens] = Q K^T, the causal mask, an fp32 online softmax in
// base 2 (one rescale of O per stage), then O[16 x D] += P V with P rounded to
// the element type.
#include "pkv_device.cuh"
#include "nvtx_range.h"
#include "pagedkv.h"
#include "tma_host.h"

#include <cuda_runtime.h>

#include <atomic>
#include <mutex>

namespace pkv {
namespace prefill {

constexpr int kWarps = 4;                    // compute warps, 16 query rows each
constexpr int kRows = kWarps * 16;           // query rows per CTA
constexpr int kThreads = (kWarps + 1) * 32;  // + the producer warp
constexpr int kBlocksPerStage = 4;           // KV blocks (64 tokens) per stage
constexpr int kStages = 3;
constexpr unsigned kFullMask = 0xffffffffu;

template <int D>
struct PGeo {
    static_assert(D == 64 || D == 128, "head dim");
    static constexpr int kTiles = D / 64;                               // 64-column boxes per block
    static constexpr int kBlockBytes = kTiles * 2048;                   // one block of one head, K or V
    static constexpr int kStageBytes = 2 * kBlocksPerStage * kBlockBytes;
    static constexpr int kRingBytes = kStages * kStageBytes;
    static constexpr int kOffBar = kRingBytes;
    static constexpr int kSmemBytes = kOffBar + 2 * kStages * 8 + 16 + 1024;  // + room to align the base
};

struct PrefillArgs {
    uint16_t *out;              // [T][Hq][D]
    const uint16_t *q;          // [T][Hq][D]
    const int32_t *block_tables;
    const int32_t *context_lens;
    const int32_t *query_start;  // [B + 1]
    int32_t *status;             // may be null
    int B, W, Hq, Hkv, group, num_blocks, max_tiles, max_query_len;
    float scale_log2;
    int slow_softmax;  // test hook: the tcgen05 path's first softmax warp hands over its first P late
    int out_f32;       // out holds fp32 numbers (a debug switch: the result before rounding)
};

__device__ __forceinline__ uint32_t swz(int row, int chunk) { return row * 128 + ((chunk ^ (row & 7)) << 4); }

__device__ __forceinline__ void flag(const PrefillArgs &a, int bits)
{
    if (a.status)
        atomicOr(a.status, bits);
}

template <class E, int D>
__global__ void __launch_bounds__(kThreads, 2) prefill_kernel(const __grid_constant__ CUtensorMap tmK,
                                                           const __grid_constant__ CUtensorMap tmV,
                                                           const PrefillArgs a)
{
    using G = PGeo<D>;
    constexpr int kBPI = D == 128 ? 2 : 4;  // KV blocks per softmax pass
    extern __shared__ unsigned char smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t ring = (raw_s + 1023u) & ~1023u;
    unsigned char *base = smem_raw + (ring - raw_s);
    uint64_t *full = reinterpret_cast<uint64_t *>(base + G::kOffBar);
    uint64_t *empty = full + kStages;
    volatile int *abort_flag = reinterpret_cast<volatile int *>(empty + kStages);
    volatile int *zero_flag = abort_flag + 1;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, j = blockIdx.y;
    const int tile = a.max_tiles - 1 - static_cast<int>(blockIdx.x);  // later rows (more KV) first
    const int g = a.group;

    // lengths and offsets: read before the grid dependency wait (the kernel
    // launched just before must not write them)
    const int q0 = __ldg(a.query_start + b);
    const int n = __ldg(a.query_start + b + 1) - q0;
    const int c = __ldg(a.context_lens + b);
    if (n <= 0)
        return;
    if (n > c || c > a.W * kBlockTokens || n > a.max_query_len) {
        if (tid == 0 && j == 0 && tile == a.max_tiles - 1) {
            grid_dependency_wait();  // the flag is the previous kernel's until then
            flag(a, KV_STATUS_BAD_CONTEXT);
        }
        return;
    }
    const int rows_total = n * g;
    const int row0 = tile * kRows;
    if (row0 >= rows_total)
        return;
    const int p0 = c - n;  // position of the chunk's first token
    const int last_row = min(row0 + kRows, rows_total) - 1;
    const int kv_len = p0 + last_row / g + 1;  // tokens this CTA reads
    const int nblk = (kv_len + kBlockTokens - 1) / kBlockTokens;
    const int nst = (nblk + kBlocksPerStage - 1) / kBlocksPerStage;

    if (tid == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);
        }
        mbar_fence_init();
        *abort_flag = 0;
        *zero_flag = 0;
    }
    __syncthreads();

    if (warp == kWarps) {
        // ---------------- producer: block ids -> TMA loads ----------------
        if (lane == 0) {
            tma_prefetch_descriptor(&tmK);
            tma_prefetch_descriptor(&tmV);
        }
        grid_dependency_wait();  // the cache may come from the kernel before (an append)
        grid_launch_dependents();
        const int32_t *row = a.block_tables + static_cast<size_t>(b) * a.W;
        int issued = 0;
        for (int st = 0; st < nst; ++st) {
            const int s = st % kStages;
            const int kb0 = st * kBlocksPerStage;
            const int nb = min(kBlocksPerStage, nblk - kb0);
            int blk = 0;
            if (lane < nb) {
                blk = __ldg(row + kb0 + lane);
                if (blk < 0 || blk >= a.num_blocks) {
                    flag(a, KV_STATUS_BAD_BLOCK_ID);
                    blk = 0;  // never read outside the pool
                }
            }
            int ok = 1;
            if (lane == 0) {
                ok = mbar_wait_bounded(&empty[s], ((st / kStages) & 1) ^ 1, abort_flag);
                if (ok)
                    mbar_arrive_expect_tx(&full[s], nb * 2 * G::kBlockBytes);
                else {
                    *abort_flag = 1;
                    flag(a, KV_STATUS_WAIT_TIMEOUT);
                }
            }
            ok = __shfl_sync(kFullMask, ok, 0);
            if (!ok)
                break;
            __syncwarp();
            if (lane < nb) {
                const uint32_t kdst = ring + s * G::kStageBytes + lane * G::kBlockBytes;
                const uint32_t vdst = kdst + kBlocksPerStage * G::kBlockBytes;
#pragma unroll
                for (int t = 0; t < G::kTiles; ++t)
                    tma_load_4d_nohint(kdst + t * 2048, &tmK, t * 64, 0, j, blk, &full[s]);
#pragma unroll
                for (int t = 0; t < G::kTiles; ++t)
                    tma_load_4d_nohint(vdst + t * 2048, &tmV, t * 64, 0, j, blk, &full[s]);
            }
            issued = st + 1;
        }
        // No load may land after this CTA exits: wait (bounded) for the last ones.
        if (lane == 0)
            for (int st = max(0, issued - kStages); st < issued; ++st)
                mbar_wait_bounded(&full[st % kStages], (st / kStages) & 1, zero_flag);
        return;
    }

    // -------------------- compute warps 0..3 --------------------
    grid_dependency_wait();  // q may come from the kernel before
    grid_launch_dependents();
    constexpr int kK = D / 16;  // k-steps of Q K^T, and pairs of 8-column tiles of O
    const int r = lane >> 2, cq = lane & 3, mi = lane >> 3, rr = lane & 7;
    const int wrow0 = row0 + warp * 16;
    const int rowA_raw = wrow0 + r, rowB_raw = rowA_raw + 8;
    const bool okA = rowA_raw < rows_total, okB = rowB_raw < rows_total;
    const int rowA = min(rowA_raw, rows_total - 1), rowB = min(rowB_raw, rows_total - 1);
    const int tokA = rowA / g, hA = rowA - tokA * g;
    const int tokB = rowB / g, hB = rowB - tokB * g;
    const int posA = p0 + tokA, posB = p0 + tokB;
    const int wlast = min(wrow0 + 15, rows_total - 1);
    const int wmin_pos = p0 + min(wrow0, rows_total - 1) / g, wmax_pos = p0 + wlast / g;

    // Q as the A operand: rows A (a0, a2) and B (a1, a3)
    uint32_t qf[kK][4];
    {
        const uint32_t *qa = reinterpret_cast<const uint32_t *>(
            a.q + (static_cast<size_t>(q0 + tokA) * a.Hq + j * g + hA) * D);
        const uint32_t *qb = reinterpret_cast<const uint32_t *>(
            a.q + (static_cast<size_t>(q0 + tokB) * a.Hq + j * g + hB) * D);
#pragma unroll
        for (int kk = 0; kk < kK; ++kk) {
            qf[kk][0] = okA ? __ldg(qa + kk * 8 + cq) : 0u;
            qf[kk][1] = okB ? __ldg(qb + kk * 8 + cq) : 0u;
            qf[kk][2] = okA ? __ldg(qa + kk * 8 + 4 + cq) : 0u;
            qf[kk][3] = okB ? __ldg(qb + kk * 8 + 4 + cq) : 0u;
        }
    }
    float o[2 * kK][4];
#pragma unroll
    for (int dt = 0; dt < 2 * kK; ++dt)
        o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;
    float mA = -INFINITY, mB = -INFINITY, lA = 0.f, lB = 0.f;
    const float sl2 = a.scale_log2;
    const int last_blk = (c - 1) / kBlockTokens;  // the sequence's last block, maybe partly filled

    for (int st = 0; st < nst; ++st) {
        const int s = st % kStages;
        if (!mbar_wait_bounded(&full[s], (st / kStages) & 1, abort_flag)) {
            if (lane == 0) {
                *abort_flag = 1;
                flag(a, KV_STATUS_WAIT_TIMEOUT);
            }
            break;
        }
        const int kb0 = st * kBlocksPerStage;
        const int tok_s = kb0 * kBlockTokens;
        // blocks of this stage that some row of this warp can see (the rest are after all of them)
        const int nbw = wmax_pos < tok_s ? 0
                                         : min(min(kBlocksPerStage, nblk - kb0), (wmax_pos - tok_s) / kBlockTokens + 1);
        const uint32_t kst0 = ring + s * G::kStageBytes;
        const uint32_t vst0 = kst0 + kBlocksPerStage * G::kBlockBytes;
#pragma unroll 1
        for (int grp = 0; grp < nbw; grp += kBPI) {
            // blocks grp .. grp + kBPI - 1 of the stage, kept to kBPI per pass to bound registers
            const uint32_t kst = kst0 + grp * G::kBlockBytes, vst = vst0 + grp * G::kBlockBytes;
            const int nbg = min(kBPI, nbw - grp);
            const int tok_g = tok_s + grp * kBlockTokens;
            const int kbg = kb0 + grp;
            // S = Q K^T: 16 rows x up to 16 * kBPI tokens, as [block][8-token tile][4]
            float sc[kBPI][2][4];
#pragma unroll
            for (int bi = 0; bi < kBPI; ++bi)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
                    sc[bi][nt][0] = sc[bi][nt][1] = sc[bi][nt][2] = sc[bi][nt][3] = 0.f;
#pragma unroll
            for (int kk = 0; kk < kK; ++kk) {
#pragma unroll
                for (int bi = 0; bi < kBPI; ++bi) {
                    if (bi < nbg) {
                        uint32_t bf[4];
                        ldmatrix_x4(bf, kst + bi * G::kBlockBytes + (kk >> 2) * 2048 +
                                            swz(((mi >> 1) << 3) + rr, ((kk & 3) << 1) + (mi & 1)));
                        E::mma(sc[bi][0], qf[kk], bf[0], bf[1]);
                        E::mma(sc[bi][1], qf[kk], bf[2], bf[3]);
                    }
                }
            }
            const bool need_mask = tok_g + nbg * kBlockTokens - 1 > wmin_pos;
            float bmA = -INFINITY, bmB = -INFINITY;
#pragma unroll
            for (int bi = 0; bi < kBPI; ++bi)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = tok_g + bi * kBlockTokens + nt * 8 + 2 * cq + (e & 1);
                        const int pos = e < 2 ? posA : posB;
                        const bool vis = bi < nbg && (!need_mask || t <= pos);
                        const float x = vis ? sc[bi][nt][e] * sl2 : -INFINITY;
                        sc[bi][nt][e] = x;
                        if (e < 2)
                            bmA = fmaxf(bmA, x);
                        else
                            bmB = fmaxf(bmB, x);
                    }
            bmA = fmaxf(bmA, __shfl_xor_sync(kFullMask, bmA, 1));
            bmA = fmaxf(bmA, __shfl_xor_sync(kFullMask, bmA, 2));
            bmB = fmaxf(bmB, __shfl_xor_sync(kFullMask, bmB, 1));
            bmB = fmaxf(bmB, __shfl_xor_sync(kFullMask, bmB, 2));
            const float nmA = fmaxf(mA, bmA), nmB = fmaxf(mB, bmB);  // finite: token 0 is in every row's range
            const float alA = exp2f(mA - nmA), alB = exp2f(mB - nmB);
            mA = nmA;
            mB = nmB;
            float sumA = 0.f, sumB = 0.f;
#pragma unroll
            for (int bi = 0; bi < kBPI; ++bi)
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    sc[bi][nt][0] = exp2f(sc[bi][nt][0] - nmA);
                    sc[bi][nt][1] = exp2f(sc[bi][nt][1] - nmA);
                    sc[bi][nt][2] = exp2f(sc[bi][nt][2] - nmB);
                    sc[bi][nt][3] = exp2f(sc[bi][nt][3] - nmB);
                    sumA += sc[bi][nt][0] + sc[bi][nt][1];
                    sumB += sc[bi][nt][2] + sc[bi][nt][3];
                }
            lA = lA * alA + sumA;
            lB = lB * alB + sumB;
#pragma unroll
            for (int dt = 0; dt < 2 * kK; ++dt) {
                o[dt][0] *= alA;
                o[dt][1] *= alA;
                o[dt][2] *= alB;
                o[dt][3] *= alB;
            }
            // O += P V, one 16-token block (the k dimension) at a time
#pragma unroll
            for (int bi = 0; bi < kBPI; ++bi) {
                if (bi < nbg) {
                    // rows of the sequence's last block past the context hold whatever the pool
                    // holds: their V halves are zeroed in the fragments so 0 * V stays 0
                    uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;  // tokens 2cq, 2cq+1 / 8+2cq, 9+2cq
                    if (kbg + bi == last_blk) {
                        const int valid = c - (tok_g + bi * kBlockTokens);  // 1..16
                        keep_lo = (2 * cq < valid ? 0x0000ffffu : 0u) | (2 * cq + 1 < valid ? 0xffff0000u : 0u);
                        keep_hi = (2 * cq + 8 < valid ? 0x0000ffffu : 0u) | (2 * cq + 9 < valid ? 0xffff0000u : 0u);
                    }
                    uint32_t pa[4];
                    pa[0] = E::pack(sc[bi][0][0], sc[bi][0][1]);
                    pa[1] = E::pack(sc[bi][0][2], sc[bi][0][3]);
                    pa[2] = E::pack(sc[bi][1][0], sc[bi][1][1]);
                    pa[3] = E::pack(sc[bi][1][2], sc[bi][1][3]);
                    const uint32_t vb = vst + bi * G::kBlockBytes;
#pragma unroll
                    for (int dp = 0; dp < kK; ++dp) {
                        uint32_t vf[4];
                        ldmatrix_x4_trans(vf, vb + (dp >> 2) * 2048 +
                                                  swz(((mi & 1) << 3) + rr, ((dp & 3) << 1) + (mi >> 1)));
                        vf[0] &= keep_lo;
                        vf[1] &= keep_hi;
                        vf[2] &= keep_lo;
                        vf[3] &= keep_hi;
                        E::mma(o[2 * dp], pa, vf[0], vf[1]);
                        E::mma(o[2 * dp + 1], pa, vf[2], vf[3]);
                    }
                }
            }
        }
        __syncwarp();
        if (lane == 0)
            mbar_arrive(&empty[s]);
    }

    // normalise and store this lane's two rows
    lA += __shfl_xor_sync(kFullMask, lA, 1);
    lA += __shfl_xor_sync(kFullMask, lA, 2);
    lB += __shfl_xor_sync(kFullMask, lB, 1);
    lB += __shfl_xor_sync(kFullMask, lB, 2);
    const float iA = 1.f / lA, iB = 1.f / lB;
    const size_t offA = (static_cast<size_t>(q0 + tokA) * a.Hq + j * g + hA) * D;
    const size_t offB = (static_cast<size_t>(q0 + tokB) * a.Hq + j * g + hB) * D;
    if (a.out_f32) {
        float2 *outA = reinterpret_cast<float2 *>(reinterpret_cast<float *>(a.out) + offA);
        float2 *outB = reinterpret_cast<float2 *>(reinterpret_cast<float *>(a.out) + offB);
#pragma unroll
        for (int dt = 0; dt < 2 * kK; ++dt) {
            if (okA)
                outA[dt * 4 + cq] = make_float2(o[dt][0] * iA, o[dt][1] * iA);
            if (okB)
                outB[dt * 4 + cq] = make_float2(o[dt][2] * iB, o[dt][3] * iB);
        }
        return;
    }
    uint32_t *outA = reinterpret_cast<uint32_t *>(a.out + offA);
    uint32_t *outB = reinterpret_cast<uint32_t *>(a.out + offB);
#pragma unroll
    for (int dt = 0; dt < 2 * kK; ++dt) {
        if (okA)
            outA[dt * 4 + cq] = E::pack(o[dt][0] * iA, o[dt][1] * iA);
        if (okB)
            outB[dt * 4 + cq] = E::pack(o[dt][2] * iB, o[dt][3] * iB);
    }
}

// ===========================================================================
// tcgen05 path. The same computation on the 5th-generation tensor cores: a CTA
// takes 128 query rows; S = Q K^T (M=128, N=64 tokens) and O += P V
// (M=128, N=D) are each a few tcgen05.mma issued by one thread, accumulating in
// tensor memory. S is double-buffered (columns 0-63 and 64-127; at D = 64 a
// third buffer sits after O): the MMAs of the next tile's S run while warps
// 0-3 turn this tile's S into P. Those warps
// own one row per thread: they read the row of S from tensor memory, run the
// online softmax (all in the thread: no shuffles) and write the row of P, as
// 16-bit pairs, over the first half of the same S buffer, where the P V MMA
// takes its A operand from. O (columns 128..) is rescaled lazily: only when a
// row's maximum grows by more than 2^8, which keeps P <= 256; the final
// division by the row sum makes the result the same as with a rescale at every
// step. Warp 4 issues the TMA tile loads, warp 5 allocates tensor memory and
// issues the MMAs. K and V have rings of their own: a K stage is free once S of
// its tile is done, so the loads of K for tile j+2 start while tile j's softmax
// and P V still run (the producer issues K two tiles ahead of V, which is also
// the order in which stages come free); with one ring for both, every S waited
// a whole load latency after the P V before it. Shared memory, 1024-byte aligned:
// Q [D/64][128 rows][128 B], then the K stages [D/64][64 tokens][128 B], then
// the V stages likewise, all 128B-swizzled (the MMA descriptors say so).
// ===========================================================================
namespace tc {

constexpr int kRows = 128;
constexpr int kThreads = 192;
constexpr int kTok = 64;               // KV tokens per tile (4 blocks)
constexpr float kRescaleLog2 = 8.f;    // rescale O when a row maximum grows by more than 2^8

// 2^x by the special-function unit's approximate base-2 exponential (results
// below 2^-126, and 2^-inf, are 0).
__device__ __forceinline__ float ex2_approx(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two fp32 lanes in one 64-bit register, for the paired arithmetic of sm_100 (fma / add .f32x2:
// one instruction for two elements), and a three-input maximum: the softmax warps are bound by
// their own instruction stream, so fewer instructions per score is what shortens a tile.
__device__ __forceinline__ unsigned long long f2pack(float lo, float hi)
{
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2unpack(unsigned long long v, float &lo, float &hi)
{
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long fma_f2(unsigned long long a, unsigned long long b, unsigned long long c)
{
    unsigned long long d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ unsigned long long add_f2(unsigned long long a, unsigned long long b)
{
    unsigned long long d;
    asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float max3(float a, float b, float c)
{
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

template <int D>
struct TGeo {
    static constexpr int kTiles = D / 64;
    static constexpr int kQBytes = kTiles * kRows * 128;
    static constexpr int kKVTileBytes = kTok * 128;              // one 64-column tile of 64 tokens
    static constexpr int kStageBytes = kTiles * kKVTileBytes;     // K (or V) of one tile
    // S buffers in tensor memory: two at D = 128 (with O they fill the CTA's 256 columns), three at
    // D = 64, where O leaves 64 columns free. S of tile j + kSBufs - 1 needs the P V of tile j - 1
    // (its buffer holds that tile's P), so a third buffer takes that P V off the path from one
    // tile's softmax to the next but one's.
    static constexpr int kSBufs = D == 64 ? 3 : 2;
    // tiles of K and of V in flight: two each at D = 128 (measured faster than three or four of K);
    // as many as S buffers at D = 64, so that the softmax of a tile (which follows S of that tile,
    // hence the P V kSBufs tiles back) never waits on a V stage two loads behind
    static constexpr int kStagesK = D == 64 ? 3 : 2;
    static constexpr int kStagesV = D == 64 ? 3 : 2;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = kOffQ + kQBytes;
    static constexpr int kOffV = kOffK + kStagesK * kStageBytes;
    static constexpr int kOffBar = kOffV + kStagesV * kStageBytes;
    // no slack for aligning the base: the buffer is declared 1024-byte aligned (checked at run time),
    // which lets two CTAs share an SM at D = 128
    // at most two CTAs per SM: two of them use all 512 tensor-memory columns (an allocation beyond
    // that would wait for a CTA to finish), so D = 64 asks for more shared memory than it uses
    // mbarriers (full and empty per K and V stage, two S buffers, two P, P V, all MMAs, Q), the TMEM
    // address and two flags
    static constexpr int kBarBytes = 256;
    static_assert((2 * kStagesK + 2 * kStagesV + 3 * kSBufs + 2) * 8 + 12 <= kBarBytes, "barrier area");
    static constexpr int kSmemBytes = kOffBar + kBarBytes < 80 * 1024 ? 80 * 1024 : kOffBar + kBarBytes;
    static constexpr int kTmemCols = 256;                       // S/P buffers at 0 and 64, O at kOCol
    static constexpr int kOCol = 128;
    // tensor-memory column of S buffer b: 0 and 64, and the third (D = 64) after O
    static __device__ __forceinline__ uint32_t scol(int b) { return b < 2 ? b * kTok : kOCol + D; }
    static_assert(kSBufs < 3 || kOCol + D + kTok <= kTmemCols, "third S buffer");
};

template <class E, int D>
__global__ void __launch_bounds__(kThreads) prefill_tc_kernel(const __grid_constant__ CUtensorMap tmK,
                                                              const __grid_constant__ CUtensorMap tmV,
                                                              const PrefillArgs a)
{
    using G = TGeo<D>;
    constexpr int kStagesK = G::kStagesK, kStagesV = G::kStagesV, kSB = G::kSBufs;
    extern __shared__ __align__(1024) unsigned char smem_tc[];
    const uint32_t base_s = smem_addr(smem_tc);
    unsigned char *base = smem_tc;
    if (base_s & 1023u) {  // the swizzle atoms need 1024-byte alignment
        if (threadIdx.x == 0) {
            grid_dependency_wait();  // the flag is the previous kernel's until then
            flag(a, KV_STATUS_BAD_CONTEXT);
        }
        return;
    }
    const uint32_t sQ = base_s + G::kOffQ, sK = base_s + G::kOffK, sV = base_s + G::kOffV;
    uint64_t *fullK = reinterpret_cast<uint64_t *>(base + G::kOffBar);
    uint64_t *emptyK = fullK + kStagesK;
    uint64_t *fullV = emptyK + kStagesK;
    uint64_t *emptyV = fullV + kStagesV;
    uint64_t *s_full = emptyV + kStagesV;  // [kSB]: one per S buffer
    // P of tile j is ready: one barrier per S buffer (tile j uses buffer j % kSB). With fewer, a warp
    // that finished a later tile could arrive again before a slower warp had arrived for tile j,
    // completing that phase early; with one per buffer, a warp's next arrival on it is for tile
    // j + kSB, which needs S of that tile, which waits for the P V of tile j
    uint64_t *p_full = s_full + kSB;
    // the P V of tile j is done: one barrier per S buffer, so that each wait (the MMA thread's before
    // it refills a buffer, a softmax warp's before it rescales O) is at most one phase behind
    uint64_t *pv_done = p_full + kSB;
    // every MMA of the CTA is done: one phase, committed once after the last P V. The epilogue cannot
    // use pv_done: while another warp is a tile behind, pv_done can be two phases short of the last,
    // and a parity wait cannot tell two phases apart
    uint64_t *o_done = pv_done + kSB;
    uint64_t *q_ready = o_done + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(q_ready + 1);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *zero_flag = abort_flag + 1;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int b = blockIdx.z, j = blockIdx.y;
    const int tile = a.max_tiles - 1 - static_cast<int>(blockIdx.x);
    const int g = a.group;
    const int q0 = __ldg(a.query_start + b);
    const int n = __ldg(a.query_start + b + 1) - q0;
    const int c = __ldg(a.context_lens + b);
    if (n <= 0)
        return;
    if (n > c || c > a.W * kBlockTokens || n > a.max_query_len) {
        if (tid == 0 && j == 0 && tile == a.max_tiles - 1) {
            grid_dependency_wait();  // the flag is the previous kernel's until then
            flag(a, KV_STATUS_BAD_CONTEXT);
        }
        return;
    }
    const int rows_total = n * g;
    const int row0 = tile * kRows;
    if (row0 >= rows_total)
        return;
    const int p0 = c - n;
    const int last_row = min(row0 + kRows, rows_total) - 1;
    const int kv_len = p0 + last_row / g + 1;
    const int nblk = (kv_len + kBlockTokens - 1) / kBlockTokens;
    const int ntiles = (kv_len + kTok - 1) / kTok;
    constexpr int fmt = E::kDtype == KV_DTYPE_BF16 ? 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < kStagesK; ++s) {
            mbar_init(&fullK[s], 1);
            mbar_init(&emptyK[s], 1);
        }
        for (int s = 0; s < kStagesV; ++s) {
            mbar_init(&fullV[s], 1);
            mbar_init(&emptyV[s], 1);
        }
        for (int b2 = 0; b2 < kSB; ++b2) {
            mbar_init(&s_full[b2], 1);
            mbar_init(&p_full[b2], kRows);
            mbar_init(&pv_done[b2], 1);
        }
        mbar_init(o_done, 1);
        mbar_init(q_ready, kRows);
        mbar_fence_init();
        *abort_flag = 0;
        *zero_flag = 0;
    }
    if (warp == 5)
        tmem_alloc(tmem_slot, G::kTmemCols);
    tcgen05_before_sync();
    __syncthreads();
    tcgen05_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ---------------- producer: block ids -> TMA loads ----------------
        if (lane == 0) {
            tma_prefetch_descriptor(&tmK);
            tma_prefetch_descriptor(&tmV);
        }
        grid_dependency_wait();
        grid_launch_dependents();
        const int32_t *trow = a.block_tables + static_cast<size_t>(b) * a.W;
        // one tile's K (which = 0) or V (which = 1): wait for its stage, then 4 blocks of TMA boxes
        auto issue = [&](int t, int which) -> bool {
            const int ns = which == 0 ? kStagesK : kStagesV;
            const int s = t % ns;
            const int nb = min(kTok / kBlockTokens, nblk - t * (kTok / kBlockTokens));
            // the tile's block ids (read again for V: the load is under the wait for the stage)
            int blk = 0;
            if (lane < nb) {
                blk = __ldg(trow + t * (kTok / kBlockTokens) + lane);
                if (blk < 0 || blk >= a.num_blocks) {
                    if (which == 0)
                        flag(a, KV_STATUS_BAD_BLOCK_ID);
                    blk = 0;
                }
            }
            uint64_t *fb = which == 0 ? &fullK[s] : &fullV[s];
            uint64_t *eb = which == 0 ? &emptyK[s] : &emptyV[s];
            int ok = 1;
            if (lane == 0) {
                ok = mbar_wait_bounded(eb, ((t / ns) & 1) ^ 1, abort_flag);
                if (ok)
                    mbar_arrive_expect_tx(fb, nb * G::kTiles * 2048);
                else {
                    *abort_flag = 1;
                    flag(a, KV_STATUS_WAIT_TIMEOUT);
                }
            }
            ok = __shfl_sync(kFullMask, ok, 0);
            if (!ok)
                return false;
            __syncwarp();
            if (lane < nb) {
                const uint32_t dst = (which == 0 ? sK : sV) + s * G::kStageBytes + lane * 2048;
                const CUtensorMap *tm = which == 0 ? &tmK : &tmV;
#pragma unroll
                for (int tt = 0; tt < G::kTiles; ++tt)
                    tma_load_4d_nohint(dst + tt * G::kKVTileBytes, tm, tt * 64, 0, j, blk, fb);
            }
            return true;
        };
        // K(0) .. K(kStagesK - 1), then V(t), K(t + kStagesK) for each t: the stages come free in
        // this order (S(t) frees K's stage, P V(t) frees V's, and the MMAs run S(t+1), P V(t), S(t+2))
        int issuedK = 0, issuedV = 0;
        bool go = true;
        for (int t = 0; t < min(kStagesK, ntiles) && go; ++t)
            if ((go = issue(t, 0)))
                issuedK = t + 1;
        for (int t = 0; t < ntiles && go; ++t) {
            if ((go = issue(t, 1)))
                issuedV = t + 1;
            if (go && t + kStagesK < ntiles && (go = issue(t + kStagesK, 0)))
                issuedK = t + kStagesK + 1;
        }
        // no load may land after this CTA exits: wait (bounded) for the last ones
        if (lane == 0) {
            for (int t = max(0, issuedK - kStagesK); t < issuedK; ++t)
                mbar_wait_bounded(&fullK[t % kStagesK], (t / kStagesK) & 1, zero_flag);
            for (int t = max(0, issuedV - kStagesV); t < issuedV; ++t)
                mbar_wait_bounded(&fullV[t % kStagesV], (t / kStagesV) & 1, zero_flag);
        }
    } else if (warp == 5) {
        // ---------------- MMA issuer (one thread) ----------------
        grid_dependency_wait();
        grid_launch_dependents();
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_f16(kRows, kTok, fmt, 0, 0);
            const uint32_t idesc_o = umma_idesc_f16(kRows, D, fmt, 0, 1);
            bool ok = mbar_wait_bounded(q_ready, 0, abort_flag);
            tcgen05_after_sync();
            // S = Q K^T for tile jt into S buffer jt % kSB
            auto issue_s = [&](int jt) -> bool {
                const int s = jt % kStagesK;
                if (!mbar_wait_bounded(&fullK[s], (jt / kStagesK) & 1, abort_flag))
                    return false;
                tcgen05_after_sync();
                const uint32_t kst = sK + s * G::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;  // 16 elements along the 128-byte row
                    const uint64_t ad = umma_desc_sw128(sQ + (kk >> 2) * (kRows * 128) + koff, 16, 1024);
                    const uint64_t bd = umma_desc_sw128(kst + (kk >> 2) * G::kKVTileBytes + koff, 16, 1024);
                    umma_f16(tmem + G::scol(jt % kSB), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[jt % kSB]);
                // S read this K stage: it may be refilled (only a refill waits for this arrival, and
                // no arrival may still be on its way when the CTA exits)
                if (jt + kStagesK < ntiles)
                    umma_commit(&emptyK[s]);
                return true;
            };
            // S of the first kSB - 1 tiles
            for (int t = 0; t < kSB - 1 && t < ntiles && ok; ++t)
                ok = issue_s(t);
            for (int jt = 0; jt < ntiles && ok; ++jt) {
                const int s = jt % kStagesV;
                const uint32_t vst = sV + s * G::kStageBytes;
                const int t = jt + kSB - 1;
                if (t < ntiles) {
                    // S of tile t goes into the buffer that P of tile t - kSB used: wait for that PV
                    if (t >= kSB && !mbar_wait_bounded(&pv_done[t % kSB], ((t - kSB) / kSB) & 1, abort_flag)) {
                        ok = false;
                        break;
                    }
                    if (!issue_s(t)) {
                        ok = false;
                        break;
                    }
                }
                if (!mbar_wait_bounded(&p_full[jt % kSB], (jt / kSB) & 1, abort_flag) ||
                    !mbar_wait_bounded(&fullV[s], (jt / kStagesV) & 1, abort_flag)) {
                    ok = false;
                    break;
                }
                tcgen05_after_sync();
                // O += P V, P (16-bit pairs) in the first 32 columns of S buffer jt % kSB
#pragma unroll
                for (int kk = 0; kk < kTok / 16; ++kk) {
                    const uint64_t bd = umma_desc_sw128(vst + kk * 2048, G::kKVTileBytes, 1024);
                    umma_f16_tmem_a(tmem + G::kOCol, tmem + G::scol(jt % kSB) + kk * 8, bd, idesc_o,
                                    (jt > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&pv_done[jt % kSB]);
                if (jt + kStagesV < ntiles)
                    umma_commit(&emptyV[s]);
            }
            if (!ok) {
                *abort_flag = 1;
                flag(a, KV_STATUS_WAIT_TIMEOUT);
            }
            // the epilogue reads O once every MMA issued here is done, and they finish before tensor
            // memory is released (below)
            umma_commit(o_done);
            mbar_wait_bounded(o_done, 0, zero_flag);
        }
        __syncwarp();
    } else {
        // ---------------- softmax: one query row per thread ----------------
        grid_dependency_wait();  // q may come from the kernel before
        grid_launch_dependents();
        const int r = tid;  // 0..127: TMEM lane and row of the tile
        const int row = row0 + r;
        const bool ok = row < rows_total;
        const int rowc = min(row, rows_total - 1);
        const int tok = rowc / g, h = rowc - tok * g;
        const int pos = p0 + tok;
        {
            const uint4 *src =
                reinterpret_cast<const uint4 *>(a.q + (static_cast<size_t>(q0 + tok) * a.Hq + j * g + h) * D);
#pragma unroll
            for (int ch = 0; ch < D / 8; ++ch) {
                const uint4 v = ok ? __ldg(src + ch) : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t dst = sQ + (ch >> 3) * (kRows * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z),
                             "r"(v.w)
                             : "memory");
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(q_ready);
        }
        const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
        const float sl2 = a.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        bool good = true;
        for (int jt = 0; jt < ntiles; ++jt) {
            // tcgen05.ld/st are warp-wide: a warp takes every branch below as one
            if (!__all_sync(kFullMask, mbar_wait_bounded(&s_full[jt % kSB], (jt / kSB) & 1, abort_flag))) {
                good = false;
                break;
            }
            tcgen05_after_sync();
            const uint32_t sbuf = lane_base + G::scol(jt % kSB);
            float x[kTok];
            {
                // the row's four loads in flight together, one wait
                uint32_t v[kTok / 16][16];
#pragma unroll
                for (int q4 = 0; q4 < kTok / 16; ++q4)
                    tmem_ld16(sbuf + q4 * 16, v[q4]);
                tmem_wait_ld();
#pragma unroll
                for (int q4 = 0; q4 < kTok / 16; ++q4)
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        x[q4 * 16 + i] = __uint_as_float(v[q4][i]);
            }
            const int tok0 = jt * kTok;
            // raw scores: tokens after this row's position are -inf (scale > 0, so the maximum of
            // the raw scores scales to the maximum of the scaled ones)
            if (tok0 + kTok - 1 > pos) {
#pragma unroll
                for (int i = 0; i < kTok; ++i)
                    x[i] = (tok0 + i <= pos) ? x[i] : -INFINITY;
            }
            // the maximum in four independent chains of three-input maxima
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < kTok; i += 2)
                mx[(i >> 1) & 3] = max3(mx[(i >> 1) & 3], x[i], x[i + 1]);
            const float rmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            const float xmax = rmax * sl2;
            bool rescale = false;
            float alpha = 1.f;
            if (xmax > m_used + kRescaleLog2) {  // always true on the first tile (m_used = -inf)
                alpha = ex2_approx(m_used - xmax);
                rescale = jt > 0;
                m_used = xmax;
                l *= alpha;
            }
            if (!rescale)
                alpha = 1.f;  // lanes that keep their scale rewrite their row unchanged
            if (__any_sync(kFullMask, rescale)) {
                // O is rescaled once the previous tile's PV has finished with it
                if (!__all_sync(kFullMask,
                                mbar_wait_bounded(&pv_done[(jt - 1) % kSB], ((jt - 1) / kSB) & 1, abort_flag))) {
                    good = false;
                    break;
                }
                tcgen05_after_sync();
                uint32_t v[16];
#pragma unroll 1
                for (int q4 = 0; q4 < D / 16; ++q4) {
                    tmem_ld16(lane_base + G::kOCol + q4 * 16, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                    tmem_st16(lane_base + G::kOCol + q4 * 16, v);
                }
                tmem_wait_st();
            }
            // scores two at a time: y = x * scale log2(e) - m (one paired FMA), P = 2^y, the row sum in
            // two paired chains
            const unsigned long long sc2 = f2pack(sl2, sl2), mm2 = f2pack(-m_used, -m_used);
            unsigned long long ps2[2] = {f2pack(0.f, 0.f), f2pack(0.f, 0.f)};
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int i0 = half * 32 + 2 * e;
                    float ya, yb;
                    f2unpack(fma_f2(f2pack(x[i0], x[i0 + 1]), sc2, mm2), ya, yb);
                    const float pa = ex2_approx(ya), pb = ex2_approx(yb);
                    ps2[e & 1] = add_f2(ps2[e & 1], f2pack(pa, pb));
                    w[e] = E::pack(pa, pb);
                }
                tmem_st16(sbuf + half * 16, w);
            }
            tmem_wait_st();
            float s0, s1, s2, s3;
            f2unpack(ps2[0], s0, s1);
            f2unpack(ps2[1], s2, s3);
            l += (s0 + s1) + (s2 + s3);
            // rows of the CTA's last tile from its last visible token on hold whatever the pool holds
            // (past the context) or whatever the stage held before (blocks not loaded): zero those V
            // rows, whose P is 0, so that 0 * V stays 0 -- once V's loads have landed (S only says
            // that K's have)
            const int vrow0 = kv_len - tok0;
            if (vrow0 < kTok) {
                if (!__all_sync(kFullMask, mbar_wait_bounded(&fullV[jt % kStagesV], (jt / kStagesV) & 1,
                                                             abort_flag))) {
                    good = false;
                    break;
                }
                const uint32_t vst = sV + (jt % kStagesV) * G::kStageBytes;
                const int cnt = (kTok - vrow0) * G::kTiles * 8;
                for (int idx = r; idx < cnt; idx += kRows) {
                    const int rr = vrow0 + idx / (G::kTiles * 8);
                    const int rem = idx % (G::kTiles * 8);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(vst + (rem >> 3) * G::kKVTileBytes +
                                                                               rr * 128 + ((rem & 7) << 4)),
                                 "r"(0)
                                 : "memory");
                }
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            tcgen05_before_sync();
            if (a.slow_softmax && warp == 0 && jt == 0) {
                // test hook: let the other warps run a tile ahead of this one (a bounded wait)
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 30000u)
                    __nanosleep(1000);
            }
            mbar_arrive(&p_full[jt % kSB]);
        }
        // epilogue: O / l
        if (__all_sync(kFullMask, good && mbar_wait_bounded(o_done, 0, abort_flag))) {
            tcgen05_after_sync();
            const float inv = 1.f / l;
            const size_t row = (static_cast<size_t>(q0 + tok) * a.Hq + j * g + h) * D;
            uint16_t *dst = a.out + row;
            uint32_t v[16];
#pragma unroll 1
            for (int q4 = 0; q4 < D / 16; ++q4) {
                tmem_ld16(lane_base + G::kOCol + q4 * 16, v);
                tmem_wait_ld();
                if (a.out_f32) {
                    if (ok) {
                        float4 *f = reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.out) + row + q4 * 16);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            f[i] = make_float4(__uint_as_float(v[4 * i]) * inv, __uint_as_float(v[4 * i + 1]) * inv,
                                               __uint_as_float(v[4 * i + 2]) * inv,
                                               __uint_as_float(v[4 * i + 3]) * inv);
                    }
                    continue;
                }
                uint4 o0, o1;
                o0.x = E::pack(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv);
                o0.y = E::pack(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv);
                o0.z = E::pack(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv);
                o0.w = E::pack(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv);
                o1.x = E::pack(__uint_as_float(v[8]) * inv, __uint_as_float(v[9]) * inv);
                o1.y = E::pack(__uint_as_float(v[10]) * inv, __uint_as_float(v[11]) * inv);
                o1.z = E::pack(__uint_as_float(v[12]) * inv, __uint_as_float(v[13]) * inv);
                o1.w = E::pack(__uint_as_float(v[14]) * inv, __uint_as_float(v[15]) * inv);
                if (ok) {
                    reinterpret_cast<uint4 *>(dst + q4 * 16)[0] = o0;
                    reinterpret_cast<uint4 *>(dst + q4 * 16)[1] = o1;
                }
            }
        } else if (lane == 0) {
            *abort_flag = 1;
            flag(a, KV_STATUS_WAIT_TIMEOUT);
        }
    }
    // every thread is past its last tensor-memory access; release it
    tcgen05_before_sync();
    __syncthreads();
    if (warp == 5) {
        tcgen05_after_sync();
        tmem_dealloc(tmem, G::kTmemCols);
    }
}

}  // namespace tc

// ===========================================================================
// tcgen05 path, two query tiles per CTA. One CTA per SM takes 256 query rows
// (two tiles of 128) and streams each 128-token K/V tile once for both. A
// tcgen05.mma of M = 128 with N = 128 runs at the tensor pipe's full rate,
// where N = 64 (the one-tile kernel's S) does not; a tile of 128 tokens also
// halves the hand-offs per flop. Tensor memory (all 512 columns of the SM):
// S of tile t at 128 t, O of tile t at 256 + D t; P of tile t is written over
// the first half of its S at D = 128 and has columns of its own at D = 64
// (384 + 64 t), where O leaves room. Warps 0-3 run the softmax of tile 0 and
// warps 4-7 that of tile 1 (one row per thread, as in the one-tile kernel),
// warp 8 issues the TMA loads, warp 9 the MMAs. At D = 128 the MMA thread
// alternates the tiles in a fixed order: while one tile's softmax runs, the
// tensor pipe does the other tile's P V and next S, which goes where P of that
// tile is and so waits for its P V. At D = 64 the next S only waits until the
// softmax has read S and runs while the softmax computes; there the MMA
// thread issues whichever tile's next S or P V is ready. CTAs start longest sequence
// first (each ranks the batch's context lengths), and the epilogue writes each
// row of O with one bulk copy from shared memory. Every hand-off is an
// mbarrier with a bounded wait, as in the one-tile kernel.
// ===========================================================================
namespace pair {

// Non-blocking test of an mbarrier phase (test_wait never suspends the thread, so one thread can watch
// several barriers in turn).
__device__ __forceinline__ bool mbar_test(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait by spinning on test_wait, for the MMA thread: false after kWaitLimitNs or once *abort is
// set. At D = 128 it hands each P V and next S over ~0.7 % faster than the suspending try_wait (on one box,
// 886-889 -> 892-895 TFLOP/s); the softmax warps spinning as well was slower (875-877): they share issue
// slots with the other tile's softmax.
__device__ __forceinline__ bool mbar_spin(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    if (mbar_test(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_test(bar, parity))
            return true;
        if ((it & 63u) == 0u && (*abort || global_timer_ns() - t0 > kWaitLimitNs))
            return false;
    }
}

constexpr int kRows = 128;     // query rows per tile; a CTA takes two
constexpr int kTok = 128;      // KV tokens per tile (8 blocks)
constexpr int kThreads = 320;  // 8 softmax warps, the producer warp, the MMA warp
constexpr int kProducerWarp = 8, kMmaWarp = 9;
constexpr int kRankMax = 256;  // batches up to this size are launched longest sequence first


template <int D>
struct Geo {
    static constexpr int kChunks = D / 64;                 // 128-byte chunks of a row of D elements
    static constexpr int kQBytes = kChunks * kRows * 128;  // one query tile
    static constexpr int kChunkBytes = kTok * 128;         // one chunk of a K or V tile
    static constexpr int kStageBytes = kChunks * kChunkBytes;
    static constexpr int kStagesK = D == 64 ? 3 : 2;
    static constexpr int kStagesV = D == 64 ? 3 : 2;
    // P in columns of its own (D = 64) or over S (D = 128, where the two O take 256 columns)
    static constexpr bool kSepP = D == 64;
    static constexpr int kOffQ = 0;
    static constexpr int kOffK = 2 * kQBytes;
    static constexpr int kOffV = kOffK + kStagesK * kStageBytes;
    static constexpr int kOffBar = kOffV + kStagesV * kStageBytes;
    // full and empty per K and V stage; per query tile S full, S read, P full, P V done and Q
    // ready; all MMAs done; the tensor-memory address and two flags
    static constexpr int kBarBytes = 256;
    static_assert((2 * kStagesK + 2 * kStagesV + 5 * 2 + 1) * 8 + 12 <= kBarBytes, "barrier area");
    static constexpr int kSmemBytes = kOffBar + kBarBytes;
    static_assert(kSmemBytes <= 227 * 1024, "shared memory");
    static constexpr int kTmemCols = 512;
    static __device__ __forceinline__ uint32_t scol(int t) { return t * kTok; }
    static __device__ __forceinline__ uint32_t ocol(int t) { return 2 * kTok + t * D; }
    static __device__ __forceinline__ uint32_t pcol(int t)
    {
        return kSepP ? 2 * kTok + 2 * D + t * (kTok / 2) : t * kTok;
    }
    static_assert(!kSepP || 2 * kTok + 2 * D + kTok <= kTmemCols, "P columns");
    static_assert(2 * kTok + 2 * D <= kTmemCols, "O columns");
};

template <class E, int D>
__global__ void __launch_bounds__(kThreads, 1) prefill_pair_kernel(const __grid_constant__ CUtensorMap tmK,
                                                                   const __grid_constant__ CUtensorMap tmV,
                                                                   const PrefillArgs a)
{
    using G = Geo<D>;
    constexpr int SK = G::kStagesK, SV = G::kStagesV;
    extern __shared__ __align__(1024) unsigned char smem_pair[];
    const uint32_t base_s = smem_addr(smem_pair);
    unsigned char *base = smem_pair;
    if (base_s & 1023u) {  // the swizzle atoms need 1024-byte alignment
        if (threadIdx.x == 0) {
            grid_dependency_wait();
            flag(a, KV_STATUS_BAD_CONTEXT);
        }
        return;
    }
    const uint32_t sQ = base_s + G::kOffQ, sK = base_s + G::kOffK, sV = base_s + G::kOffV;
    uint64_t *fullK = reinterpret_cast<uint64_t *>(base + G::kOffBar);
    uint64_t *emptyK = fullK + SK;
    uint64_t *fullV = emptyK + SK;
    uint64_t *emptyV = fullV + SV;
    uint64_t *s_full = emptyV + SV;  // [2]: S of the tile's current KV tile is in tensor memory
    uint64_t *s_read = s_full + 2;   // [2]: the softmax has read it (used with P apart from S)
    uint64_t *p_full = s_read + 2;   // [2]: P is in tensor memory (and the last V rows zeroed)
    uint64_t *pv_done = p_full + 2;  // [2]: O += P V is done
    uint64_t *o_done = pv_done + 2;  // every MMA of the CTA is done (one phase)
    uint64_t *q_ready = o_done + 1;  // [2]
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(q_ready + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    volatile int *zero_flag = abort_flag + 1;

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    // grid: x the kv head, y the pair of query tiles (later rows, which see more KV, first), z the
    // sequence's rank by context length (longest first, ties by index). CTAs start in that order, so
    // with one CTA per SM the long ones do not wait for the short ones' SMs at the end of the launch
    int b = blockIdx.z;
    if (a.B <= kRankMax) {
        __shared__ int s_lens[kRankMax];
        __shared__ int s_seq;
        for (int i = tid; i < a.B; i += kThreads)
            s_lens[i] = __ldg(a.context_lens + i);
        __syncthreads();
        for (int i = tid; i < a.B; i += kThreads) {
            const int ci = s_lens[i];
            int rank = 0;
            for (int k = 0; k < a.B; ++k)
                rank += (s_lens[k] > ci || (s_lens[k] == ci && k < i)) ? 1 : 0;
            if (rank == static_cast<int>(blockIdx.z))  // the ranks are a permutation: one writer
                s_seq = i;
        }
        __syncthreads();
        b = s_seq;
    }
    const int j = blockIdx.x;
    const int tile = a.max_tiles - 1 - static_cast<int>(blockIdx.y);  // pair of query tiles
    const int g = a.group;
    const int q0 = __ldg(a.query_start + b);
    const int n = __ldg(a.query_start + b + 1) - q0;
    const int c = __ldg(a.context_lens + b);
    if (n <= 0)
        return;
    if (n > c || c > a.W * kBlockTokens || n > a.max_query_len) {
        if (tid == 0 && j == 0 && tile == a.max_tiles - 1) {
            grid_dependency_wait();
            flag(a, KV_STATUS_BAD_CONTEXT);
        }
        return;
    }
    const int rows_total = n * g;
    const int row0 = tile * 2 * kRows;
    if (row0 >= rows_total)
        return;
    const int p0 = c - n;
    const int last_row = min(row0 + 2 * kRows, rows_total) - 1;
    const int kv_len = p0 + last_row / g + 1;
    const int nblk = (kv_len + kBlockTokens - 1) / kBlockTokens;
    const int ntiles = (kv_len + kTok - 1) / kTok;
    constexpr int fmt = E::kDtype == KV_DTYPE_BF16 ? 1 : 0;

    if (tid == 0) {
        for (int s = 0; s < SK; ++s) {
            mbar_init(&fullK[s], 1);
            mbar_init(&emptyK[s], 1);
        }
        for (int s = 0; s < SV; ++s) {
            mbar_init(&fullV[s], 1);
            mbar_init(&emptyV[s], 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(&s_full[t], 1);
            mbar_init(&s_read[t], kRows);
            mbar_init(&p_full[t], kRows);
            mbar_init(&pv_done[t], 1);
            mbar_init(&q_ready[t], kRows);
        }
        mbar_init(o_done, 1);
        mbar_fence_init();
        *abort_flag = 0;
        *zero_flag = 0;
    }
    if (warp == kMmaWarp)
        tmem_alloc(tmem_slot, G::kTmemCols);
    tcgen05_before_sync();
    __syncthreads();
    tcgen05_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == kProducerWarp) {
        // ---------------- producer: block ids -> TMA loads ----------------
        if (lane == 0) {
            tma_prefetch_descriptor(&tmK);
            tma_prefetch_descriptor(&tmV);
        }
        grid_dependency_wait();
        grid_launch_dependents();
        const int32_t *trow = a.block_tables + static_cast<size_t>(b) * a.W;
        constexpr int kBlk = kTok / kBlockTokens;
        // K (which = 0) or V (which = 1) of KV tile t: wait for its stage, then one lane per block
        auto issue = [&](int t, int which) -> bool {
            const int ns = which == 0 ? SK : SV;
            const int s = t % ns;
            const int nb = min(kBlk, nblk - t * kBlk);
            int blk = 0;
            if (lane < nb) {
                blk = __ldg(trow + t * kBlk + lane);
                if (blk < 0 || blk >= a.num_blocks) {
                    if (which == 0)
                        flag(a, KV_STATUS_BAD_BLOCK_ID);
                    blk = 0;
                }
            }
            uint64_t *fb = which == 0 ? &fullK[s] : &fullV[s];
            uint64_t *eb = which == 0 ? &emptyK[s] : &emptyV[s];
            int ok = 1;
            if (lane == 0) {
                ok = mbar_wait_bounded(eb, ((t / ns) & 1) ^ 1, abort_flag);
                if (ok)
                    mbar_arrive_expect_tx(fb, nb * G::kChunks * 2048);
                else {
                    *abort_flag = 1;
                    flag(a, KV_STATUS_WAIT_TIMEOUT);
                }
            }
            ok = __shfl_sync(kFullMask, ok, 0);
            if (!ok)
                return false;
            __syncwarp();
            if (lane < nb) {
                const uint32_t dst = (which == 0 ? sK : sV) + s * G::kStageBytes + lane * 2048;
                const CUtensorMap *tm = which == 0 ? &tmK : &tmV;
#pragma unroll
                for (int ch = 0; ch < G::kChunks; ++ch)
                    tma_load_4d_nohint(dst + ch * G::kChunkBytes, tm, ch * 64, 0, j, blk, fb);
            }
            return true;
        };
        // K(t), V(t) for each t: the order in which the MMAs need them and free their stages
        int issuedK = 0, issuedV = 0;
        bool go = true;
        for (int t = 0; t < ntiles && go; ++t) {
            if ((go = issue(t, 0)))
                issuedK = t + 1;
            if (go && (go = issue(t, 1)))
                issuedV = t + 1;
        }
        // no load may land after this CTA exits: wait (bounded) for the last ones
        if (lane == 0) {
            for (int t = max(0, issuedK - SK); t < issuedK; ++t)
                mbar_wait_bounded(&fullK[t % SK], (t / SK) & 1, zero_flag);
            for (int t = max(0, issuedV - SV); t < issuedV; ++t)
                mbar_wait_bounded(&fullV[t % SV], (t / SV) & 1, zero_flag);
        }
    } else if (warp == kMmaWarp) {
        // ---------------- MMA issuer (one thread) ----------------
        grid_dependency_wait();
        grid_launch_dependents();
        if (lane == 0) {
            const uint32_t idesc_s = umma_idesc_f16(kRows, kTok, fmt, 0, 0);
            const uint32_t idesc_o = umma_idesc_f16(kRows, D, fmt, 0, 1);
            // S of query tile t for KV tile jt: Q_t K^T into its S columns
            auto issue_s = [&](int jt, int t) {
                const uint32_t kst = sK + (jt % SK) * G::kStageBytes;
                const uint32_t qt = sQ + t * G::kQBytes;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk & 3) * 32;  // 16 elements along the 128-byte row
                    const uint64_t ad = umma_desc_sw128(qt + (kk >> 2) * (kRows * 128) + koff, 16, 1024);
                    const uint64_t bd = umma_desc_sw128(kst + (kk >> 2) * G::kChunkBytes + koff, 16, 1024);
                    umma_f16(tmem + G::scol(t), ad, bd, idesc_s, kk > 0 ? 1u : 0u);
                }
                umma_commit(&s_full[t]);
            };
            // O_t += P_t V for KV tile jt, P (16-bit pairs) read from tensor memory
            auto issue_pv = [&](int jt, int t) {
                const uint32_t vst = sV + (jt % SV) * G::kStageBytes;
#pragma unroll
                for (int kk = 0; kk < kTok / 16; ++kk) {
                    const uint64_t bd = umma_desc_sw128(vst + kk * 2048, G::kChunkBytes, 1024);
                    umma_f16_tmem_a(tmem + G::ocol(t), tmem + G::pcol(t) + kk * 8, bd, idesc_o,
                                    (jt > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit(&pv_done[t]);
            };
            // Issue order at D = 128 (P over S): per KV tile, tile 0's P V and next S, then tile 1's. This keeps
            // the two softmaxes about half a cycle apart, so they take turns on the special-function units;
            // issuing whatever is ready first (watching both tiles' barriers) let them drift into step and ran
            // 20 % slower there. At D = 64 the next S does not wait for a P V, and ready-first is the order.
            bool ok = mbar_wait_bounded(&q_ready[0], 0, abort_flag) && mbar_wait_bounded(&fullK[0], 0, abort_flag);
            if (ok) {
                tcgen05_after_sync();
                issue_s(0, 0);
                ok = mbar_wait_bounded(&q_ready[1], 0, abort_flag);
            }
            if (ok) {
                tcgen05_after_sync();
                issue_s(0, 1);
                if (SK < ntiles)  // only a refill waits for this arrival
                    umma_commit(&emptyK[0]);
            }
            if (G::kSepP) {
                // P apart from S (D = 64): whichever tile's next MMA is ready goes first. S(j + 1) of a tile
                // needs only that its softmax has read S(j) and that K(j + 1) has landed, P V(j) that P(j)
                // is full and V(j) has landed; in a fixed order (per KV tile, tile 0's MMAs, then tile 1's) a
                // tile's next S waited behind the other tile's P (a timestamp trace: ~1,160 cycles of each
                // ~3,280-cycle query-tile cycle spent waiting for S). A K or V stage is released by a commit after the second of the
                // two tiles' MMAs that read it; tile 1's P V of the last KV tile follows tile 0's, whose
                // P-full arrival comes after the zeroing of that tile's V rows past the context.
                int ns[2] = {1, 1};  // next S per tile (S of KV tile 0 went out above)
                int np[2] = {0, 0};  // next P V per tile
                uint64_t since = global_timer_ns();
                uint32_t idle = 0;
                while (ok && (np[0] < ntiles || np[1] < ntiles)) {
                    bool moved = false;
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int js = ns[t];
                        if (js < ntiles && mbar_test(&s_read[t], (js - 1) & 1) &&
                            mbar_test(&fullK[js % SK], (js / SK) & 1)) {
                            tcgen05_after_sync();
                            issue_s(js, t);
                            if (ns[t ^ 1] > js && js + SK < ntiles)
                                umma_commit(&emptyK[js % SK]);
                            ns[t] = js + 1;
                            moved = true;
                        }
                        const int jp = np[t];
                        if (jp < ntiles && !(t == 1 && jp == ntiles - 1 && np[0] < ntiles) &&
                            mbar_test(&p_full[t], jp & 1) && mbar_test(&fullV[jp % SV], (jp / SV) & 1)) {
                            tcgen05_after_sync();
                            issue_pv(jp, t);
                            if (np[t ^ 1] > jp && jp + SV < ntiles)
                                umma_commit(&emptyV[jp % SV]);
                            np[t] = jp + 1;
                            moved = true;
                        }
                    }
                    if (moved) {
                        idle = 0;
                        since = global_timer_ns();
                    } else if ((++idle & 63u) == 0u && (*abort_flag || global_timer_ns() - since > kWaitLimitNs)) {
                        ok = false;  // nothing became ready for a whole wait limit (or another warp gave up)
                    }
                }
            }
            // P over S (D = 128), a fixed order: per KV tile, tile 0's P V and next S, then tile 1's
            for (int jt = 0; jt < ntiles && ok && !G::kSepP; ++jt) {
                const bool more = jt + 1 < ntiles;
                const int kn = (jt + 1) % SK;
                for (int t = 0; t < 2 && ok; ++t) {
                    if (!mbar_spin(&p_full[t], jt & 1, abort_flag) ||
                        (t == 0 && !mbar_spin(&fullV[jt % SV], (jt / SV) & 1, abort_flag))) {
                        ok = false;
                        break;
                    }
                    tcgen05_after_sync();
                    issue_pv(jt, t);
                    if (t == 1 && jt + SV < ntiles)
                        umma_commit(&emptyV[jt % SV]);
                    if (more) {
                        // the next S overwrites this P: after its P V
                        if ((t == 0 && !mbar_spin(&fullK[kn], ((jt + 1) / SK) & 1, abort_flag)) ||
                            !mbar_spin(&pv_done[t], jt & 1, abort_flag)) {
                            ok = false;
                            break;
                        }
                        tcgen05_after_sync();
                        issue_s(jt + 1, t);
                        if (t == 1 && jt + 1 + SK < ntiles)
                            umma_commit(&emptyK[kn]);
                    }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                flag(a, KV_STATUS_WAIT_TIMEOUT);
            }
            umma_commit(o_done);
            mbar_wait_bounded(o_done, 0, zero_flag);
        }
        __syncwarp();
    } else {
        // ---------------- softmax: warps 4t..4t+3 own query tile t, one row per thread ----------------
        grid_dependency_wait();  // q may come from the kernel before
        grid_launch_dependents();
        const int t = warp >> 2;
        const int r = tid & (kRows - 1);  // TMEM lane and row of the tile
        const int row = row0 + t * kRows + r;
        const bool ok = row < rows_total;
        const int rowc = min(row, rows_total - 1);
        const int tok = rowc / g, h = rowc - tok * g;
        const int pos = p0 + tok;
        {
            const uint32_t qt = sQ + t * G::kQBytes;
            const uint4 *src =
                reinterpret_cast<const uint4 *>(a.q + (static_cast<size_t>(q0 + tok) * a.Hq + j * g + h) * D);
#pragma unroll
            for (int ch = 0; ch < D / 8; ++ch) {
                const uint4 v = ok ? __ldg(src + ch) : make_uint4(0u, 0u, 0u, 0u);
                const uint32_t dst = qt + (ch >> 3) * (kRows * 128) + r * 128 + (((ch & 7) ^ (r & 7)) << 4);
                asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(v.x), "r"(v.y), "r"(v.z),
                             "r"(v.w)
                             : "memory");
            }
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            mbar_arrive(&q_ready[t]);
        }
        const uint32_t lane_base = tmem + (static_cast<uint32_t>((warp & 3) * 32) << 16);
        const float sl2 = a.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        bool good = true;
        for (int jt = 0; jt < ntiles; ++jt) {
            // tcgen05.ld/st are warp-wide: a warp takes every branch below as one
            if (!__all_sync(kFullMask, mbar_wait_bounded(&s_full[t], jt & 1, abort_flag))) {
                good = false;
                break;
            }
            tcgen05_after_sync();
            float x[kTok];
            {
                // the row's eight loads in flight together, one wait (reading the row in two halves, each
                // twice, held fewer registers but ran 7 % slower)
                uint32_t v[kTok / 16][16];
#pragma unroll
                for (int q8 = 0; q8 < kTok / 16; ++q8)
                    tmem_ld16(lane_base + G::scol(t) + q8 * 16, v[q8]);
                tmem_wait_ld();
#pragma unroll
                for (int q8 = 0; q8 < kTok / 16; ++q8)
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        x[q8 * 16 + i] = __uint_as_float(v[q8][i]);
            }
            if (G::kSepP) {
                tcgen05_before_sync();
                mbar_arrive(&s_read[t]);  // the next S may be written over these columns
            }
            const int tok0 = jt * kTok;
            if (tok0 + kTok - 1 > pos) {  // tokens after this row's position are -inf
#pragma unroll
                for (int i = 0; i < kTok; ++i)
                    x[i] = (tok0 + i <= pos) ? x[i] : -INFINITY;
            }
            // the maximum of the raw scores in four chains of three-input maxima (scale > 0, so it scales to
            // the maximum of the scaled ones)
            float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
            for (int i = 0; i < kTok; i += 2)
                mx[(i >> 1) & 3] = tc::max3(mx[(i >> 1) & 3], x[i], x[i + 1]);
            const float rmax = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
            const float xmax = rmax * sl2;
            bool rescale = false;
            float alpha = 1.f;
            if (xmax > m_used + tc::kRescaleLog2) {  // always true on the first tile (m_used = -inf)
                alpha = tc::ex2_approx(m_used - xmax);
                rescale = jt > 0;
                m_used = xmax;
                l *= alpha;
            }
            if (!rescale)
                alpha = 1.f;
            const bool any_rescale = __any_sync(kFullMask, rescale);
            // O is rescaled, and (P apart from S) P rewritten, once the previous P V is done with them;
            // with P over S that is already so: S of this tile was issued after it
            if (jt > 0 && (any_rescale || G::kSepP)) {
                if (!__all_sync(kFullMask, mbar_wait_bounded(&pv_done[t], (jt - 1) & 1, abort_flag))) {
                    good = false;
                    break;
                }
                tcgen05_after_sync();
            }
            if (any_rescale) {
                uint32_t v[16];
#pragma unroll 1
                for (int q4 = 0; q4 < D / 16; ++q4) {
                    tmem_ld16(lane_base + G::ocol(t) + q4 * 16, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
                    tmem_st16(lane_base + G::ocol(t) + q4 * 16, v);
                }
                tmem_wait_st();
            }
            // P = 2^(x scale log2(e) - m_used), two scores at a time (one paired FMA), on the special-
            // function unit (computing part of them with a polynomial on the FMA pipe instead, and computing
            // P against the running maximum before the tile's own maximum was known, both measured slower);
            // the row sum in four paired chains
            const unsigned long long sc2 = tc::f2pack(sl2, sl2), mm2 = tc::f2pack(-m_used, -m_used);
            unsigned long long ps2[4] = {tc::f2pack(0.f, 0.f), tc::f2pack(0.f, 0.f), tc::f2pack(0.f, 0.f),
                                         tc::f2pack(0.f, 0.f)};
#pragma unroll
            for (int qq = 0; qq < kTok / 32; ++qq) {
                uint32_t w[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int i0 = qq * 32 + 2 * e;
                    float ya, yb;
                    tc::f2unpack(tc::fma_f2(tc::f2pack(x[i0], x[i0 + 1]), sc2, mm2), ya, yb);
                    const float pa = tc::ex2_approx(ya), pb = tc::ex2_approx(yb);
                    ps2[e & 3] = tc::add_f2(ps2[e & 3], tc::f2pack(pa, pb));
                    w[e] = E::pack(pa, pb);
                }
                tmem_st16(lane_base + G::pcol(t) + qq * 16, w);
            }
            tmem_wait_st();
            {
                float s0, s1, s2, s3, s4, s5, s6, s7;
                tc::f2unpack(ps2[0], s0, s1);
                tc::f2unpack(ps2[1], s2, s3);
                tc::f2unpack(ps2[2], s4, s5);
                tc::f2unpack(ps2[3], s6, s7);
                l += ((s0 + s1) + (s2 + s3)) + ((s4 + s5) + (s6 + s7));
            }
            // rows of the last KV tile from the CTA's last visible token on hold whatever the pool
            // holds past the context, or what the stage held before: tile 0's warps zero those V rows
            // (P is 0 there, and 0 * V must stay 0) once V's loads have landed; tile 1's P V is issued
            // after tile 0's P is full, so after the zeroing
            const int vrow0 = kv_len - tok0;
            if (t == 0 && vrow0 < kTok) {
                if (!__all_sync(kFullMask, mbar_wait_bounded(&fullV[jt % SV], (jt / SV) & 1, abort_flag))) {
                    good = false;
                    break;
                }
                const uint32_t vst = sV + (jt % SV) * G::kStageBytes;
                const int cnt = (kTok - vrow0) * G::kChunks * 8;
                for (int idx = r; idx < cnt; idx += kRows) {
                    const int rr = vrow0 + idx / (G::kChunks * 8);
                    const int rem = idx % (G::kChunks * 8);
                    asm volatile("st.shared.v4.b32 [%0], {%1,%1,%1,%1};" ::"r"(vst + (rem >> 3) * G::kChunkBytes +
                                                                               rr * 128 + ((rem & 7) << 4)),
                                 "r"(0)
                                 : "memory");
                }
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the P V reads these zeros
            }
            tcgen05_before_sync();
            if (a.slow_softmax && warp == 0 && jt == 0) {
                // test hook: let the other warps run ahead of this one (a bounded wait)
                const uint64_t t0 = global_timer_ns();
                while (global_timer_ns() - t0 < 30000u)
                    __nanosleep(1000);
            }
            mbar_arrive(&p_full[t]);
        }
        // epilogue: O / l. The tile's four warps decide together (a warp that gave up must not leave the
        // others at a barrier)
        const bool done = mbar_wait_bounded(o_done, 0, abort_flag);
        if (named_barrier_and(1 + t, kRows, good && done)) {
            tcgen05_after_sync();
            const float inv = 1.f / l;
            if (a.out_f32) {
                const size_t orow = (static_cast<size_t>(q0 + tok) * a.Hq + j * g + h) * D;
                uint32_t v[16];
#pragma unroll 1
                for (int q4 = 0; q4 < D / 16; ++q4) {
                    tmem_ld16(lane_base + G::ocol(t) + q4 * 16, v);
                    tmem_wait_ld();
                    if (ok) {
                        float4 *f = reinterpret_cast<float4 *>(reinterpret_cast<float *>(a.out) + orow + q4 * 16);
#pragma unroll
                        for (int i = 0; i < 4; ++i)
                            f[i] = make_float4(__uint_as_float(v[4 * i]) * inv, __uint_as_float(v[4 * i + 1]) * inv,
                                               __uint_as_float(v[4 * i + 2]) * inv,
                                               __uint_as_float(v[4 * i + 3]) * inv);
                    }
                }
            } else {
                // Each thread's row goes to shared memory (the K/V stages: every MMA is done with them) and out
                // with one bulk copy, issued by the thread itself: a row of O per thread stored directly would
                // make every warp store touch 32 rows. Rows are padded to 2D + 16 bytes, so that the 32 rows a
                // warp writes at once fall on different banks.
                constexpr int kPitch = 2 * D + 16;
                static_assert(2 * kRows * kPitch <= (G::kStagesK + G::kStagesV) * G::kStageBytes, "staging");
                const uint32_t srow = sK + (t * kRows + r) * kPitch;
                const size_t orow = (static_cast<size_t>(q0 + tok) * a.Hq + j * g + h) * D;
                uint32_t v[16];
#pragma unroll 1
                for (int q4 = 0; q4 < D / 16; ++q4) {
                    tmem_ld16(lane_base + G::ocol(t) + q4 * 16, v);
                    tmem_wait_ld();
                    // columns i, i + 1 of the row, scaled, as one word of two 16-bit elements
                    auto word = [&](int i) {
                        return E::pack(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv);
                    };
#pragma unroll
                    for (int hlf = 0; hlf < 2; ++hlf)
                        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(srow + q4 * 32 + hlf * 16),
                                     "r"(word(8 * hlf)), "r"(word(8 * hlf + 2)), "r"(word(8 * hlf + 4)),
                                     "r"(word(8 * hlf + 6))
                                     : "memory");
                }
                if (ok) {
                    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // the copy reads these writes
                    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(a.out + orow),
                                 "r"(srow), "n"(2 * D)
                                 : "memory");
                    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                    // the copy has read the row before the CTA (and its shared memory) is gone
                    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
                }
            }
        } else if (lane == 0) {
            *abort_flag = 1;
            flag(a, KV_STATUS_WAIT_TIMEOUT);
        }
    }
    // every thread is past its last tensor-memory access; release it
    tcgen05_before_sync();
    __syncthreads();
    if (warp == kMmaWarp) {
        tcgen05_after_sync();
        tmem_dealloc(tmem, G::kTmemCols);
    }
}

}  // namespace pair
}  // namespace prefill
}  // namespace pkv

// KV_OPT_PREFILL_PATH and KV_OPT_TEST_SLOW_SOFTMAX, kept with the other switches in decode.cu
int pkv_prefill_path();
int pkv_prefill_slow_softmax();
int pkv_out_f32();

namespace {

using PrefillFn = void (*)(const CUtensorMap, const CUtensorMap, const pkv::prefill::PrefillArgs);

PrefillFn pick_prefill_tc(int dtype, int D, int *smem)
{
    using namespace pkv;
    using namespace pkv::prefill::tc;
    *smem = D == 64 ? TGeo<64>::kSmemBytes : TGeo<128>::kSmemBytes;
    if (dtype == KV_DTYPE_FP16)
        return D == 64 ? prefill_tc_kernel<ElemF16, 64> : prefill_tc_kernel<ElemF16, 128>;
    return D == 64 ? prefill_tc_kernel<ElemBf16, 64> : prefill_tc_kernel<ElemBf16, 128>;
}

PrefillFn pick_prefill_pair(int dtype, int D, int *smem)
{
    using namespace pkv;
    using namespace pkv::prefill::pair;
    *smem = D == 64 ? Geo<64>::kSmemBytes : Geo<128>::kSmemBytes;
    if (dtype == KV_DTYPE_FP16)
        return D == 64 ? prefill_pair_kernel<ElemF16, 64> : prefill_pair_kernel<ElemF16, 128>;
    return D == 64 ? prefill_pair_kernel<ElemBf16, 64> : prefill_pair_kernel<ElemBf16, 128>;
}

PrefillFn pick_prefill(int dtype, int D, int *smem)
{
    using namespace pkv;
    using namespace pkv::prefill;
    *smem = D == 64 ? PGeo<64>::kSmemBytes : PGeo<128>::kSmemBytes;
    if (dtype == KV_DTYPE_FP16)
        return D == 64 ? prefill_kernel<ElemF16, 64> : prefill_kernel<ElemF16, 128>;
    return D == 64 ? prefill_kernel<ElemBf16, 64> : prefill_kernel<ElemBf16, 128>;
}

bool prepare_prefill(PrefillFn fn, int smem, int dev)
{
    struct Entry {
        const void *fn;
        int dev;
    };
    static std::mutex mu;
    static Entry done[16];
    static int used = 0;
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i)
        if (done[i].fn == reinterpret_cast<const void *>(fn) && done[i].dev == dev)
            return true;
    if (cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
        return false;
    if (used < 16)
        done[used++] = Entry{reinterpret_cast<const void *>(fn), dev};
    return true;
}

bool misaligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; }

}  // namespace

extern "C" kv_status paged_attention_prefill(void *out, const void *q, const void *k_cache, const void *v_cache,
                                             const int32_t *block_tables, int max_blocks_per_seq,
                                             const int32_t *context_lens, const int32_t *query_start, int B,
                                             int max_query_len, int num_blocks, int Hq, int Hkv, int D, float scale,
                                             int dtype, int32_t *error_flag, kv_stream_t stream)
{
    pkv_host::NvtxRange nvtx_range("paged_attention_prefill");
    using namespace pkv::prefill;
    if ((dtype != KV_DTYPE_BF16 && dtype != KV_DTYPE_FP16) || B < 0 || B > 65535 || max_query_len < 0 ||
        max_blocks_per_seq < 1 || num_blocks < 1 || Hq < 1 || Hkv < 1 || Hkv > 65535 || Hq % Hkv != 0 ||
        (D != 64 && D != 128))
        return KV_ERR_ARG;
    if (B == 0 || max_query_len == 0)
        return KV_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !query_start)
        return KV_ERR_ARG;
    if (misaligned16(out) || misaligned16(q) || misaligned16(k_cache) || misaligned16(v_cache))
        return KV_ERR_ARG;
    const int group = Hq / Hkv;
    if (!(scale > 0.f))
        return KV_ERR_ARG;
    // 1: tcgen05, one query tile per CTA; 2: mma.sync; 3 (and auto): tcgen05, two query tiles per CTA
    const int path = pkv_prefill_path() == 0 ? 3 : pkv_prefill_path();
    const int rows_per_cta = path == 3 ? 2 * pair::kRows : path == 1 ? tc::kRows : kRows;
    const long long tiles = (static_cast<long long>(max_query_len) * group + rows_per_cta - 1) / rows_per_cta;
    if (tiles > (path == 3 ? 65535ll : (1ll << 31) - 1))
        return KV_ERR_ARG;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess)
        return KV_ERR_CUDA;
    int smem = 0;
    PrefillFn fn = path == 3 ? pick_prefill_pair(dtype, D, &smem)
                   : path == 1 ? pick_prefill_tc(dtype, D, &smem)
                               : pick_prefill(dtype, D, &smem);
    if (!prepare_prefill(fn, smem, dev))
        return KV_ERR_CUDA;
    CUtensorMap tmK, tmV;
    if (!pkv_host::make_cache_map(&tmK, k_cache, num_blocks, Hkv, D, 1, dtype) ||
        !pkv_host::make_cache_map(&tmV, v_cache, num_blocks, Hkv, D, 1, dtype))
        return KV_ERR_CUDA;
    PrefillArgs a;
    a.out = static_cast<uint16_t *>(out);
    a.q = static_cast<const uint16_t *>(q);
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.query_start = query_start;
    a.status = error_flag;
    a.B = B;
    a.W = max_blocks_per_seq;
    a.Hq = Hq;
    a.Hkv = Hkv;
    a.group = group;
    a.num_blocks = num_blocks;
    a.max_tiles = static_cast<int>(tiles);
    a.max_query_len = max_query_len;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.slow_softmax = pkv_prefill_slow_softmax();
    a.out_f32 = pkv_out_f32();

    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = path == 3 ? dim3(static_cast<unsigned>(Hkv), static_cast<unsigned>(tiles), static_cast<unsigned>(B))
                            : dim3(static_cast<unsigned>(tiles), static_cast<unsigned>(Hkv), static_cast<unsigned>(B));
    cfg.blockDim = dim3(path == 3 ? pair::kThreads : path == 1 ? tc::kThreads : kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, fn, tmK, tmV, a) == cudaSuccess ? KV_OK : KV_ERR_CUDA;
}

/*
 * Float64 CPU oracle for one decode step of attention over a paged KV cache.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the bench's CPU-baseline leg
 * do. It shares no code, header, table or constant with the CUDA library.
 *
 * What it computes is the plain definition, written out step by step:
 *
 *   - "Module 23: Serving", section 23.4 (Paged Attention): the cache lives in
 *     fixed-size blocks of 16 tokens, and a per-sequence table maps logical
 *     positions to physical blocks.  Token t of sequence b therefore sits in
 *     physical block block_tables[b][t / 16], row t % 16.
 *   - "Scaling LLM serving", section "The KV cache" (Share key/value heads):
 *     grouped-query attention, a group of query heads shares one key/value
 *     head.  Groups are contiguous: query head h reads kv head h / (Hq / Hkv).
 *   - "Module 23: Serving", section 23.2 (Prefill and Decode): decode reads the
 *     whole KV cache for one new token per sequence, i.e. for every query head
 *     out = softmax(scale * q K^T) V over all c cached tokens.
 *
 * Layouts (all row-major, element type noted):
 *   q            [B][Hq][D]                    bf16 bit patterns (uint16)
 *   k_cache      [num_blocks][16][Hkv][D]      bf16 bit patterns
 *   v_cache      [num_blocks][16][Hkv][D]      bf16 bit patterns
 *   (oracle_paged_attention_decode_fp16: the same with IEEE binary16 bit
 *   patterns; "Module 23: Serving", section 23.1: 2 bytes per number for
 *   fp16 or bf16)
 *   block_tables [B][W]                        int32 physical block ids
 *   context_lens [B]                           int32 tokens cached (>= 0)
 *   out          [B][Hq][D]                    float64
 *   weight_sums  [B][Hq] (optional)            float64, sum of softmax weights
 *
 * context_len = 0 is defined as out = 0 (no token to attend to).
 *
 * Return value: 0 on success, -1 on an argument error (bad shape, a context
 * longer than the table row, a block id outside [0, num_blocks)), -2 when a
 * scratch allocation fails.  Nothing is written to out on error.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_BLOCK_TOKENS 16

/* bf16 is the upper half of an IEEE binary32; widening it to double is exact. */
static double bf16_bits_to_double(uint16_t bits)
{
    uint32_t word = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &word, sizeof f);
    return (double)f;
}

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
 * Exponent 0 holds zero and the subnormals (fraction * 2^-24), exponent 31
 * infinity (fraction 0) and NaN. Every value is exact in double. */
static double fp16_bits_to_double(uint16_t bits)
{
    const int sign = bits >> 15;
    const int expo = (bits >> 10) & 0x1f;
    const int frac = bits & 0x3ff;
    double mag;
    if (expo == 0)
        mag = ldexp((double)frac, -24);
    else if (expo == 31)
        mag = frac ? NAN : INFINITY;
    else
        mag = ldexp((double)(1024 + frac), expo - 25);
    return sign ? -mag : mag;
}

/* Step 1 of the definition: where logical token t of sequence b lives. */
static size_t cache_row_offset(const int32_t *block_tables, int W, int b, int t,
                               int Hkv, int j, int D)
{
    int32_t phys = block_tables[(size_t)b * W + t / ORACLE_BLOCK_TOKENS];
    int row = t % ORACLE_BLOCK_TOKENS;
    return (((size_t)phys * ORACLE_BLOCK_TOKENS + row) * Hkv + j) * (size_t)D;
}

static int decode_any(double *out, double *weight_sums,
                      const uint16_t *q,
                      const uint16_t *k_cache,
                      const uint16_t *v_cache,
                      const int32_t *block_tables, int W,
                      const int32_t *context_lens, int B,
                      int num_blocks, int Hq, int Hkv, int D,
                      double scale, double (*widen)(uint16_t))
{
    if (B < 0 || W < 0 || Hq <= 0 || Hkv <= 0 || D <= 0 || num_blocks < 0)
        return -1;
    if (Hq % Hkv != 0)
        return -1;
    /* Validate every table entry that will be read before touching anything. */
    for (int b = 0; b < B; ++b) {
        int c = context_lens[b];
        if (c < 0 || c > W * ORACLE_BLOCK_TOKENS)
            return -1;
        int nblk = (c + ORACLE_BLOCK_TOKENS - 1) / ORACLE_BLOCK_TOKENS;
        for (int i = 0; i < nblk; ++i) {
            int32_t phys = block_tables[(size_t)b * W + i];
            if (phys < 0 || phys >= num_blocks)
                return -1;
        }
    }

    const int group = Hq / Hkv;
    int failed = 0;

#pragma omp parallel for schedule(dynamic, 1)
    for (long bh = 0; bh < (long)B * Hq; ++bh) {
        const int b = (int)(bh / Hq);
        const int h = (int)(bh % Hq);
        const int j = h / group;            /* kv head shared by this group */
        const int c = context_lens[b];
        double *o = out + (size_t)bh * D;

        for (int d = 0; d < D; ++d)
            o[d] = 0.0;
        if (weight_sums)
            weight_sums[bh] = 0.0;
        if (c == 0)
            continue;

        double *z = (double *)malloc((size_t)c * sizeof(double));
        if (!z) {
#pragma omp atomic write
            failed = 1;
            continue;
        }

        /* Step 2: logits z_t = scale * <q_h, K_t>, all in float64. */
        const uint16_t *qh = q + (size_t)bh * D;
        for (int t = 0; t < c; ++t) {
            const uint16_t *kt = k_cache + cache_row_offset(block_tables, W, b, t, Hkv, j, D);
            double dot = 0.0;
            for (int d = 0; d < D; ++d)
                dot += widen(qh[d]) * widen(kt[d]);
            z[t] = scale * dot;
        }

        /* Step 3: softmax weights, shifted by the maximum logit. */
        double zmax = z[0];
        for (int t = 1; t < c; ++t)
            if (z[t] > zmax)
                zmax = z[t];
        double denom = 0.0;
        for (int t = 0; t < c; ++t) {
            z[t] = exp(z[t] - zmax);
            denom += z[t];
        }

        /* Step 4: out = sum_t w_t V_t. */
        double wsum = 0.0;
        for (int t = 0; t < c; ++t) {
            const double w = z[t] / denom;
            const uint16_t *vt = v_cache + cache_row_offset(block_tables, W, b, t, Hkv, j, D);
            for (int d = 0; d < D; ++d)
                o[d] += w * widen(vt[d]);
            wsum += w;
        }
        if (weight_sums)
            weight_sums[bh] = wsum;
        free(z);
    }
    return failed ? -2 : 0;
}

int oracle_paged_attention_decode(double *out, double *weight_sums,
                                  const uint16_t *q,
                                  const uint16_t *k_cache,
                                  const uint16_t *v_cache,
                                  const int32_t *block_tables, int W,
                                  const int32_t *context_lens, int B,
                                  int num_blocks, int Hq, int Hkv, int D,
                                  double scale)
{
    return decode_any(out, weight_sums, q, k_cache, v_cache, block_tables, W, context_lens, B,
                      num_blocks, Hq, Hkv, D, scale, bf16_bits_to_double);
}

int oracle_paged_attention_decode_fp16(double *out, double *weight_sums,
                                       const uint16_t *q,
                                       const uint16_t *k_cache,
                                       const uint16_t *v_cache,
                                       const int32_t *block_tables, int W,
                                       const int32_t *context_lens, int B,
                                       int num_blocks, int Hq, int Hkv, int D,
                                       double scale)
{
    return decode_any(out, weight_sums, q, k_cache, v_cache, block_tables, W, context_lens, B,
                      num_blocks, Hq, Hkv, D, scale, fp16_bits_to_double);
}

/* Widening of one bit pattern (kind 0: bf16, 1: fp16), exposed so the tests can
 * check the conversions against an independent library over all 65536 codes. */
double oracle_widen(int kind, uint16_t bits)
{
    return kind ? fp16_bits_to_double(bits) : bf16_bits_to_double(bits);
}

/*
 * Append oracle ("Module 23: Serving", section 23.4: blocks are filled as the
 * sequence grows).  For every i with slot_mapping[i] >= 0, the new token's
 * K and V rows for all Hkv heads are copied byte for byte into
 *   cache[slot / 16][slot % 16][:][:].
 * Negative slots are padding and are skipped.  Slots must be distinct.
 * Returns -1 (and writes nothing) if any slot is >= num_blocks * 16.
 */
int oracle_kv_cache_append(uint16_t *k_cache, uint16_t *v_cache,
                           const uint16_t *k_new, const uint16_t *v_new,
                           const int64_t *slot_mapping, int T,
                           int num_blocks, int Hkv, int D)
{
    const int64_t limit = (int64_t)num_blocks * ORACLE_BLOCK_TOKENS;
    for (int i = 0; i < T; ++i)
        if (slot_mapping[i] >= limit)
            return -1;
    const size_t row = (size_t)Hkv * D;
    for (int i = 0; i < T; ++i) {
        const int64_t slot = slot_mapping[i];
        if (slot < 0)
            continue;
        const int64_t blk = slot / ORACLE_BLOCK_TOKENS;
        const int64_t off = slot % ORACLE_BLOCK_TOKENS;
        const size_t dst = ((size_t)blk * ORACLE_BLOCK_TOKENS + (size_t)off) * row;
        memcpy(k_cache + dst, k_new + (size_t)i * row, row * sizeof(uint16_t));
        memcpy(v_cache + dst, v_new + (size_t)i * row, row * sizeof(uint16_t));
    }
    return 0;
}

/* Threads the OpenMP runtime will use for the attention loop. */
int oracle_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

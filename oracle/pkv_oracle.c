/*
 * pkv_oracle.c -- the float64 CPU oracle for paged KV-cache decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library,
 * its C ABI or the Python binding) may include, link or call this file.  Only
 * the tests, the smoke check and the CPU-baseline leg of the benchmark use it.
 * It shares no code, header, table or constant with the CUDA sources.
 *
 * What it follows (the pages carry no code; each function restates the plain
 * definition the pages describe):
 *
 *  - "vLLM 深读：用 PagedAttention 撑起高并发 LLM 推理" (ai-maas.com INS-0007),
 *    section "先看浪费在哪里": the KV cache is cut into fixed-size blocks that
 *    are logically contiguous and physically scattered, a block table maps one
 *    to the other, and shared prefix blocks are reference counted with
 *    copy-on-write.
 *  - ipipp.com vLLM article, section "二、PagedAttention分页原理深度剖析":
 *    16 tokens per block by default; a per-sequence block table maps logical
 *    to physical blocks; the kernel visits the sequence block by block, looks
 *    up the physical block, loads it and computes; the result is the same
 *    attention as over contiguous memory.
 *  - "vLLM" wiki entry (wiki.bytelighting.cn), section "Flattened 布局与
 *    slot_mapping": slot_mapping maps a logical token position to a physical
 *    slot of the flattened cache.
 *
 * Readings where the pages are silent (each is listed in the design notes):
 *  - cache layout [num_blocks][num_kv_heads][block_size][head_dim] for K and
 *    for V separately;
 *  - query head h reads kv head h / (num_q_heads / num_kv_heads);
 *  - attention is plain softmax(scale * q.K^T) V over the whole context, the
 *    context length including the token being decoded;
 *  - an empty context (length 0) yields a zero output;
 *  - a negative slot marks a padding token and is skipped;
 *  - copy_blocks reads every source before writing any destination.
 *
 * Every float input (fp32 or bf16) is widened exactly to double; all
 * arithmetic is double, exp() is libm's.
 *
 * Pins: tests/test_oracle_pins.py checks this file against dense attention,
 * closed forms, hand-derived fixtures (tests/golden/) and the paging
 * invariants (placement permutation, shared vs private prefix, poisoned
 * padding, partition associativity).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* Status codes returned by the oracle (0 = ok). */
enum {
    ORACLE_OK = 0,
    ORACLE_BAD_ARG = 1,
    ORACLE_BAD_BLOCK = 2,   /* a block-table entry inside the context is out of range */
    ORACLE_BAD_LEN = 3,     /* context length negative or beyond the table */
    ORACLE_BAD_SLOT = 4,    /* slot beyond the pool */
    ORACLE_BAD_PAIR = 5,    /* copy pair out of range */
    ORACLE_NO_MEMORY = 6
};

enum { ORACLE_F32 = 0, ORACLE_BF16 = 1, ORACLE_E4M3 = 2, ORACLE_E5M2 = 3 };

static int is_fp8(int dtype)
{
    return dtype == ORACLE_E4M3 || dtype == ORACLE_E5M2;
}

/* ------------------------------------------------------------------------- */
/* FP8 E4M3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
 * infinities; exponent 15 with mantissa 7 is NaN, so the largest finite value
 * is 1.75 * 2^8 = 448; exponent 0 holds the subnormals m * 2^-9).  A KV cache
 * in this format stores code = e4m3(x / scale) with one scale per pool; the
 * reading of "quantise" used here: divide in single precision, round to the
 * nearest representable value with ties to even, saturate to +-448 instead of
 * overflowing, keep NaN. */
static double e4m3_value(uint8_t code)
{
    const int sign = code >> 7, exp = (code >> 3) & 15, man = code & 7;
    double v;
    if (exp == 15 && man == 7) {
        return NAN;
    }
    if (exp == 0) {
        v = ldexp((double)man, -9);
    } else {
        v = ldexp(1.0 + man / 8.0, exp - 7);
    }
    return sign ? -v : v;
}

static uint8_t e4m3_encode(float y)
{
    if (isnan(y)) {
        return 0x7f;
    }
    const uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a >= 448.0) {
        return sign | 0x7e;                       /* saturate */
    }
    int e;
    frexp(a, &e);                                 /* a = f * 2^e, 0.5 <= f < 1 */
    int unbiased = e - 1;                         /* a in [2^unbiased, 2^(unbiased+1)) */
    if (a == 0.0 || unbiased < -6) {
        unbiased = -6;                            /* subnormal range: steps of 2^-9 */
    }
    /* number of 2^(unbiased-3) steps, rounded to nearest, ties to even (rint
     * under the default rounding mode) */
    double steps = rint(ldexp(a, 3 - unbiased));
    if (steps >= 16.0) {                          /* rounded up into the next binade */
        unbiased += 1;
        steps = 8.0;
    }
    if (unbiased > 8 || (unbiased == 8 && steps > 14.0)) {
        return sign | 0x7e;                       /* beyond 448 after rounding */
    }
    if (steps < 8.0) {                            /* subnormal */
        return sign | (uint8_t)steps;
    }
    return sign | (uint8_t)(((unbiased + 7) << 3) | ((int)steps - 8));
}

/* FP8 E5M2 (1 sign bit, 5 exponent bits with bias 15, 2 mantissa bits, the
 * IEEE-style layout of the upper byte of a binary16: exponent 31 holds the
 * infinities (mantissa 0) and NaNs, so the largest finite value is
 * 1.75 * 2^15 = 57344; exponent 0 holds the subnormals m * 2^-16).  The same
 * reading of "quantise" as for e4m3: divide in single precision, round to the
 * nearest representable value with ties to even, saturate to +-57344 instead
 * of overflowing, keep NaN. */
static double e5m2_value(uint8_t code)
{
    const int sign = code >> 7, exp = (code >> 2) & 31, man = code & 3;
    double v;
    if (exp == 31) {
        v = man == 0 ? INFINITY : NAN;
    } else if (exp == 0) {
        v = ldexp((double)man, -16);
    } else {
        v = ldexp(1.0 + man / 4.0, exp - 15);
    }
    return sign ? -v : v;
}

static uint8_t e5m2_encode(float y)
{
    if (isnan(y)) {
        return 0x7f;
    }
    const uint8_t sign = signbit(y) ? 0x80 : 0x00;
    double a = fabs((double)y);
    if (a >= 57344.0) {
        return sign | 0x7b;                       /* saturate (infinities too) */
    }
    int e;
    frexp(a, &e);                                 /* a = f * 2^e, 0.5 <= f < 1 */
    int unbiased = e - 1;                         /* a in [2^unbiased, 2^(unbiased+1)) */
    if (a == 0.0 || unbiased < -14) {
        unbiased = -14;                           /* subnormal range: steps of 2^-16 */
    }
    /* number of 2^(unbiased-2) steps, rounded to nearest, ties to even */
    double steps = rint(ldexp(a, 2 - unbiased));
    if (steps >= 8.0) {                           /* rounded up into the next binade */
        unbiased += 1;
        steps = 4.0;
    }
    if (unbiased > 15) {
        return sign | 0x7b;                       /* beyond 57344 after rounding */
    }
    if (steps < 4.0) {                            /* subnormal */
        return sign | (uint8_t)steps;
    }
    return sign | (uint8_t)(((unbiased + 15) << 2) | ((int)steps - 4));
}

/* Encode n floats: out[i] = e5m2(x[i] / scale), the division in float. */
int oracle_e5m2_quantize(const float *x, int64_t n, float scale, uint8_t *out)
{
    if ((!x || !out) && n > 0) {
        return 1;
    }
    for (int64_t i = 0; i < n; ++i) {
        out[i] = e5m2_encode(x[i] / scale);
    }
    return 0;
}

/* Decode n e5m2 codes to doubles (exact values, without any scale). */
int oracle_e5m2_values(const uint8_t *codes, int64_t n, double *out)
{
    if ((!codes || !out) && n > 0) {
        return 1;
    }
    for (int64_t i = 0; i < n; ++i) {
        out[i] = e5m2_value(codes[i]);
    }
    return 0;
}

/* Encode n floats: out[i] = e4m3(x[i] / scale), the division in float. */
int oracle_e4m3_quantize(const float *x, int64_t n, float scale, uint8_t *out)
{
    if ((!x || !out) && n > 0) {
        return 1;
    }
    for (int64_t i = 0; i < n; ++i) {
        out[i] = e4m3_encode(x[i] / scale);
    }
    return 0;
}

/* Decode n codes to doubles (the exact values, without any scale). */
int oracle_e4m3_values(const uint8_t *codes, int64_t n, double *out)
{
    if ((!codes || !out) && n > 0) {
        return 1;
    }
    for (int64_t i = 0; i < n; ++i) {
        out[i] = e4m3_value(codes[i]);
    }
    return 0;
}

/* Widen one stored element to double.  bf16 is the upper half of an IEEE
 * binary32, so shifting its 16 bits up gives the exact float, and float to
 * double is exact.  An e4m3 code widens to its exact value (the pool's scale
 * is applied by the caller). */
static double widen(const void *base, int64_t index, int dtype)
{
    if (dtype == ORACLE_F32) {
        return (double)((const float *)base)[index];
    }
    if (dtype == ORACLE_E4M3) {
        return e4m3_value(((const uint8_t *)base)[index]);
    }
    if (dtype == ORACLE_E5M2) {
        return e5m2_value(((const uint8_t *)base)[index]);
    }
    uint32_t bits = (uint32_t)((const uint16_t *)base)[index] << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

/* ------------------------------------------------------------------------- */
/* Slot indexing.  Token position j of a sequence lives in logical block
 * j / block_size at offset j % block_size; the block table gives the physical
 * block, and the slot is that block's first slot plus the offset. */
int oracle_slot_mapping(const int32_t *block_tables, int32_t max_blocks_per_seq,
                        int32_t block_size, const int32_t *token_seq,
                        const int32_t *token_pos, int32_t num_tokens,
                        int64_t *slots)
{
    if (!block_tables || !token_seq || !token_pos || !slots || block_size <= 0 ||
        max_blocks_per_seq <= 0 || num_tokens < 0) {
        return ORACLE_BAD_ARG;
    }
    for (int32_t t = 0; t < num_tokens; ++t) {
        int32_t seq = token_seq[t];
        int32_t pos = token_pos[t];
        if (seq < 0 || pos < 0 || pos / block_size >= max_blocks_per_seq) {
            return ORACLE_BAD_ARG;
        }
        int64_t logical_block = pos / block_size;
        int64_t offset = pos % block_size;
        int64_t physical_block =
            block_tables[(int64_t)seq * max_blocks_per_seq + logical_block];
        slots[t] = physical_block * block_size + offset;
    }
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* reshape_and_cache: the new K and V of token t ([t][kv_head][d] rows) are
 * written verbatim into the cache at slot_mapping[t].  No conversion. */
int oracle_reshape_and_cache(const void *k, const void *v, void *k_cache,
                             void *v_cache, const int64_t *slot_mapping,
                             int32_t num_tokens, int32_t num_kv_heads,
                             int32_t head_dim, int32_t elem_bytes,
                             int32_t block_size, int64_t num_blocks)
{
    if (!k || !v || !k_cache || !v_cache || !slot_mapping || num_tokens < 0 ||
        num_kv_heads <= 0 || head_dim <= 0 || elem_bytes <= 0 || block_size <= 0 ||
        num_blocks <= 0) {
        return ORACLE_BAD_ARG;
    }
    const size_t row = (size_t)head_dim * (size_t)elem_bytes;
    int status = ORACLE_OK;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) {
            continue; /* padding token */
        }
        if (slot >= num_blocks * block_size) {
            status = ORACLE_BAD_SLOT;
            continue;
        }
        int64_t block = slot / block_size;
        int64_t offset = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            size_t src = ((size_t)t * num_kv_heads + h) * row;
            size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) * row;
            memcpy((char *)k_cache + dst, (const char *)k + src, row);
            memcpy((char *)v_cache + dst, (const char *)v + src, row);
        }
    }
    return status;
}

/* reshape_and_cache into FP8 (e4m3) pools: token t's bf16 K and V values are
 * quantised (code = e4m3(value / scale), the division in float) and written
 * at slot_mapping[t]. */
static int reshape_and_cache_f8(const uint16_t *k, const uint16_t *v, uint8_t *k_cache,
                                uint8_t *v_cache, const int64_t *slot_mapping,
                                int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int64_t num_blocks, float k_scale,
                                float v_scale, uint8_t (*encode)(float));

int oracle_reshape_and_cache_fp8(const uint16_t *k, const uint16_t *v, uint8_t *k_cache,
                                 uint8_t *v_cache, const int64_t *slot_mapping,
                                 int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                 int32_t block_size, int64_t num_blocks, float k_scale,
                                 float v_scale)
{
    return reshape_and_cache_f8(k, v, k_cache, v_cache, slot_mapping, num_tokens,
                                num_kv_heads, head_dim, block_size, num_blocks, k_scale,
                                v_scale, e4m3_encode);
}

/* The same into e5m2 pools: code = e5m2(value / scale). */
int oracle_reshape_and_cache_e5m2(const uint16_t *k, const uint16_t *v, uint8_t *k_cache,
                                  uint8_t *v_cache, const int64_t *slot_mapping,
                                  int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                  int32_t block_size, int64_t num_blocks, float k_scale,
                                  float v_scale)
{
    return reshape_and_cache_f8(k, v, k_cache, v_cache, slot_mapping, num_tokens,
                                num_kv_heads, head_dim, block_size, num_blocks, k_scale,
                                v_scale, e5m2_encode);
}

static int reshape_and_cache_f8(const uint16_t *k, const uint16_t *v, uint8_t *k_cache,
                                uint8_t *v_cache, const int64_t *slot_mapping,
                                int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                                int32_t block_size, int64_t num_blocks, float k_scale,
                                float v_scale, uint8_t (*encode)(float))
{
    if (!k || !v || !k_cache || !v_cache || !slot_mapping || num_tokens < 0 ||
        num_kv_heads <= 0 || head_dim <= 0 || block_size <= 0 || num_blocks <= 0) {
        return ORACLE_BAD_ARG;
    }
    int status = ORACLE_OK;
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) {
            continue;
        }
        if (slot >= num_blocks * block_size) {
            status = ORACLE_BAD_SLOT;
            continue;
        }
        int64_t block = slot / block_size, offset = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            for (int32_t d = 0; d < head_dim; ++d) {
                size_t src = ((size_t)t * num_kv_heads + h) * head_dim + d;
                size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) *
                                 head_dim + d;
                k_cache[dst] = encode((float)widen(k, (int64_t)src, ORACLE_BF16) / k_scale);
                v_cache[dst] = encode((float)widen(v, (int64_t)src, ORACLE_BF16) / v_scale);
            }
        }
    }
    return status;
}

/* ------------------------------------------------------------------------- */
/* copy_blocks: for each pair (src, dst) the whole K block and the whole V block
 * of src (all kv heads, all slots) are copied to dst.  Sources are taken from a
 * snapshot made before any write, so the result does not depend on pair order. */
int oracle_copy_blocks(void *k_cache, void *v_cache, const int64_t *pairs,
                       int32_t num_pairs, int64_t block_bytes, int64_t num_blocks)
{
    if (!k_cache || !v_cache || (!pairs && num_pairs > 0) || num_pairs < 0 ||
        block_bytes <= 0 || num_blocks <= 0) {
        return ORACLE_BAD_ARG;
    }
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
            return ORACLE_BAD_PAIR;
        }
    }
    if (num_pairs == 0) {
        return ORACLE_OK;
    }
    char *snap_k = malloc((size_t)num_pairs * (size_t)block_bytes);
    char *snap_v = malloc((size_t)num_pairs * (size_t)block_bytes);
    if (!snap_k || !snap_v) {
        free(snap_k);
        free(snap_v);
        return ORACLE_NO_MEMORY;
    }
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t src = pairs[2 * i];
        memcpy(snap_k + (size_t)i * block_bytes,
               (const char *)k_cache + (size_t)src * block_bytes, (size_t)block_bytes);
        memcpy(snap_v + (size_t)i * block_bytes,
               (const char *)v_cache + (size_t)src * block_bytes, (size_t)block_bytes);
    }
    for (int32_t i = 0; i < num_pairs; ++i) {
        int64_t dst = pairs[2 * i + 1];
        memcpy((char *)k_cache + (size_t)dst * block_bytes,
               snap_k + (size_t)i * block_bytes, (size_t)block_bytes);
        memcpy((char *)v_cache + (size_t)dst * block_bytes,
               snap_v + (size_t)i * block_bytes, (size_t)block_bytes);
    }
    free(snap_k);
    free(snap_v);
    return ORACLE_OK;
}

/* ------------------------------------------------------------------------- */
/* Paged decode attention. */

typedef struct {
    const void *q, *k_cache, *v_cache;
    int dtype;
    const int32_t *block_tables, *context_lens;
    int32_t num_seqs, num_q_heads, num_kv_heads, head_dim, block_size;
    int64_t num_blocks;
    int32_t max_blocks_per_seq;
    double scale;
    /* FP8 caches: q is bf16, each cache element is code * its pool's scale */
    double k_scale, v_scale;
} problem;

static int q_dtype(const problem *pb)
{
    return is_fp8(pb->dtype) ? ORACLE_BF16 : pb->dtype;
}

/* Gather the contiguous K and V rows [0, len) of (seq, kv_head) by walking the
 * block table one logical block at a time.  Returns ORACLE_BAD_BLOCK if an
 * entry the context needs is out of range. */
static int gather_context(const problem *pb, int32_t seq, int32_t kv_head,
                          int32_t len, double *K, double *V)
{
    const int32_t D = pb->head_dim;
    for (int32_t j = 0; j < len; ++j) {
        int32_t logical_block = j / pb->block_size;
        int32_t offset = j % pb->block_size;
        int64_t physical_block =
            pb->block_tables[(int64_t)seq * pb->max_blocks_per_seq + logical_block];
        if (physical_block < 0 || physical_block >= pb->num_blocks) {
            return ORACLE_BAD_BLOCK;
        }
        int64_t row =
            ((physical_block * pb->num_kv_heads + kv_head) * pb->block_size + offset) * D;
        for (int32_t d = 0; d < D; ++d) {
            K[(int64_t)j * D + d] = widen(pb->k_cache, row + d, pb->dtype) * pb->k_scale;
            V[(int64_t)j * D + d] = widen(pb->v_cache, row + d, pb->dtype) * pb->v_scale;
        }
    }
    return ORACLE_OK;
}

/* Plain softmax attention of one query row over tokens [t0, t1) of the
 * gathered K/V.  Writes m = max score, l = sum of exp(score - m) and
 * o = sum_j exp(score_j - m) V_j / l.  An empty range gives m = -inf, l = 0,
 * o = 0. */
static void attend_range(const double *qrow, const double *K, const double *V,
                         int32_t D, double scale, int32_t t0, int32_t t1,
                         double *m_out, double *l_out, double *o)
{
    for (int32_t d = 0; d < D; ++d) {
        o[d] = 0.0;
    }
    if (t1 <= t0) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return;
    }
    double *z = malloc(sizeof(double) * (size_t)(t1 - t0));
    double m = -INFINITY;
    for (int32_t j = t0; j < t1; ++j) {
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d) {
            dot += qrow[d] * K[(int64_t)j * D + d];
        }
        z[j - t0] = scale * dot;
        if (z[j - t0] > m) {
            m = z[j - t0];
        }
    }
    double l = 0.0;
    for (int32_t j = t0; j < t1; ++j) {
        double w = exp(z[j - t0] - m);
        l += w;
        for (int32_t d = 0; d < D; ++d) {
            o[d] += w * V[(int64_t)j * D + d];
        }
    }
    for (int32_t d = 0; d < D; ++d) {
        o[d] /= l;
    }
    *m_out = m;
    *l_out = l;
    free(z);
}

/* Check the context length of a sequence against the table width. */
static int checked_len(const problem *pb, int32_t seq, int32_t *len)
{
    int32_t L = pb->context_lens[seq];
    if (L < 0 || (int64_t)L > (int64_t)pb->max_blocks_per_seq * pb->block_size) {
        return ORACLE_BAD_LEN;
    }
    *len = L;
    return ORACLE_OK;
}

/* One (seq, q_head) task: out[0:D] = softmax(scale q.K^T) V over the context. */
static int decode_one(const problem *pb, int32_t seq, int32_t q_head, double *out)
{
    const int32_t D = pb->head_dim;
    const int32_t group = pb->num_q_heads / pb->num_kv_heads;
    const int32_t kv_head = q_head / group;
    int32_t L;
    int st = checked_len(pb, seq, &L);
    if (st != ORACLE_OK) {
        return st;
    }
    double *qrow = malloc(sizeof(double) * (size_t)D);
    double *K = malloc(sizeof(double) * ((size_t)L * D + 1));
    double *V = malloc(sizeof(double) * ((size_t)L * D + 1));
    if (!qrow || !K || !V) {
        free(qrow);
        free(K);
        free(V);
        return ORACLE_NO_MEMORY;
    }
    for (int32_t d = 0; d < D; ++d) {
        qrow[d] = widen(pb->q, ((int64_t)seq * pb->num_q_heads + q_head) * D + d, q_dtype(pb));
    }
    st = gather_context(pb, seq, kv_head, L, K, V);
    if (st == ORACLE_OK) {
        double m, l;
        attend_range(qrow, K, V, D, pb->scale, 0, L, &m, &l, out);
    }
    free(qrow);
    free(K);
    free(V);
    return st;
}

typedef struct {
    const problem *pb;
    double *out;
    const int32_t *tasks; /* (seq, q_head) pairs, or NULL for all */
    int64_t num_tasks;
    int64_t next;         /* shared task counter */
    int status;           /* first error seen */
} task_pool;

static void *decode_worker(void *arg)
{
    task_pool *tp = arg;
    const problem *pb = tp->pb;
    for (;;) {
        int64_t i = __atomic_fetch_add(&tp->next, 1, __ATOMIC_RELAXED);
        if (i >= tp->num_tasks) {
            break;
        }
        int32_t seq, q_head;
        if (tp->tasks) {
            seq = tp->tasks[2 * i];
            q_head = tp->tasks[2 * i + 1];
        } else {
            seq = (int32_t)(i / pb->num_q_heads);
            q_head = (int32_t)(i % pb->num_q_heads);
        }
        int st = decode_one(pb, seq, q_head, tp->out + i * pb->head_dim);
        if (st != ORACLE_OK) {
            int expected = ORACLE_OK;
            __atomic_compare_exchange_n(&tp->status, &expected, st, 0,
                                        __ATOMIC_RELAXED, __ATOMIC_RELAXED);
        }
    }
    return NULL;
}

static int paged_decode_scaled(double *out, const void *q, const void *k_cache,
                               const void *v_cache, int32_t dtype, float k_scale, float v_scale,
                               const int32_t *block_tables, const int32_t *context_lens,
                               int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t block_size, int64_t num_blocks,
                               int32_t max_blocks_per_seq, float scale,
                               const int32_t *tasks, int64_t num_tasks, int32_t num_threads);

/*
 * out: [num_tasks][head_dim] doubles.  With tasks == NULL every (seq, q_head)
 * is computed in row-major order (num_tasks must then be num_seqs*num_q_heads),
 * else tasks holds num_tasks (seq, q_head) pairs.  num_threads <= 0 means 1.
 */
int oracle_paged_decode(double *out, const void *q, const void *k_cache,
                        const void *v_cache, int32_t dtype,
                        const int32_t *block_tables, const int32_t *context_lens,
                        int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                        int32_t head_dim, int32_t block_size, int64_t num_blocks,
                        int32_t max_blocks_per_seq, float scale,
                        const int32_t *tasks, int64_t num_tasks, int32_t num_threads)
{
    return paged_decode_scaled(out, q, k_cache, v_cache, dtype, 1.0f, 1.0f, block_tables,
                               context_lens, num_seqs, num_q_heads, num_kv_heads, head_dim,
                               block_size, num_blocks, max_blocks_per_seq, scale, tasks,
                               num_tasks, num_threads);
}

/* The same for an FP8 (e4m3) cache: q is bf16; each cached element is its
 * code's value times k_scale (K pool) or v_scale (V pool). */
int oracle_paged_decode_fp8(double *out, const void *q, const void *k_cache,
                            const void *v_cache, float k_scale, float v_scale,
                            const int32_t *block_tables, const int32_t *context_lens,
                            int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t block_size, int64_t num_blocks,
                            int32_t max_blocks_per_seq, float scale,
                            const int32_t *tasks, int64_t num_tasks, int32_t num_threads)
{
    return paged_decode_scaled(out, q, k_cache, v_cache, ORACLE_E4M3, k_scale, v_scale,
                               block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
                               head_dim, block_size, num_blocks, max_blocks_per_seq, scale,
                               tasks, num_tasks, num_threads);
}

static int paged_decode_scaled(double *out, const void *q, const void *k_cache,
                               const void *v_cache, int32_t dtype, float k_scale, float v_scale,
                               const int32_t *block_tables, const int32_t *context_lens,
                               int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                               int32_t head_dim, int32_t block_size, int64_t num_blocks,
                               int32_t max_blocks_per_seq, float scale,
                               const int32_t *tasks, int64_t num_tasks, int32_t num_threads)
{
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens ||
        (dtype != ORACLE_F32 && dtype != ORACLE_BF16 && !is_fp8(dtype)) ||
        num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 ||
        num_q_heads % num_kv_heads != 0 || head_dim <= 0 || block_size <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq <= 0 || num_tasks < 0) {
        return ORACLE_BAD_ARG;
    }
    if (!tasks && num_tasks != (int64_t)num_seqs * num_q_heads) {
        return ORACLE_BAD_ARG;
    }
    if (tasks) {
        for (int64_t i = 0; i < num_tasks; ++i) {
            if (tasks[2 * i] < 0 || tasks[2 * i] >= num_seqs || tasks[2 * i + 1] < 0 ||
                tasks[2 * i + 1] >= num_q_heads) {
                return ORACLE_BAD_ARG;
            }
        }
    }
    problem pb = {q, k_cache, v_cache, dtype, block_tables, context_lens,
                  num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                  num_blocks, max_blocks_per_seq, (double)scale, (double)k_scale,
                  (double)v_scale};
    task_pool tp = {&pb, out, tasks, num_tasks, 0, ORACLE_OK};
    if (num_threads <= 1) {
        decode_worker(&tp);
        return tp.status;
    }
    pthread_t *threads = malloc(sizeof(pthread_t) * (size_t)num_threads);
    if (!threads) {
        return ORACLE_NO_MEMORY;
    }
    int started = 0;
    for (int i = 0; i < num_threads; ++i) {
        if (pthread_create(&threads[i], NULL, decode_worker, &tp) != 0) {
            break;
        }
        ++started;
    }
    if (started == 0) {
        decode_worker(&tp);
    }
    for (int i = 0; i < started; ++i) {
        pthread_join(threads[i], NULL);
    }
    free(threads);
    return tp.status;
}

/* ------------------------------------------------------------------------- */
/* Several query tokens per sequence (a chunk of new tokens, e.g. speculative
 * tokens being verified or a slice of a prompt).  The chunk of sequence s is
 * q rows query_start_loc[s] .. query_start_loc[s+1]-1; its i-th token sits at
 * position L - n + i (L = context_lens[s] includes the chunk, n = chunk
 * length) and attends causally: to keys j <= L - n + i.  The layout of the
 * flattened query rows follows the wiki's "Flattened 布局与 slot_mapping"
 * (cu_seqlens separate the requests); causality is the plain reading of
 * autoregressive attention.  With n = 1 this is oracle_paged_decode. */
typedef struct {
    const problem *pb;
    const int32_t *query_start_loc;
    double *out;
    int64_t next;
    int status;
} multi_pool;

static void *multi_worker(void *arg)
{
    multi_pool *mp = arg;
    const problem *pb = mp->pb;
    const int32_t D = pb->head_dim;
    const int32_t group = pb->num_q_heads / pb->num_kv_heads;
    for (;;) {
        int64_t task = __atomic_fetch_add(&mp->next, 1, __ATOMIC_RELAXED);
        if (task >= (int64_t)pb->num_seqs * pb->num_kv_heads) {
            break;
        }
        int32_t seq = (int32_t)(task / pb->num_kv_heads);
        int32_t kv_head = (int32_t)(task % pb->num_kv_heads);
        int32_t L, st;
        st = checked_len(pb, seq, &L);
        int32_t q0 = mp->query_start_loc[seq], n = mp->query_start_loc[seq + 1] - q0;
        if (st == ORACLE_OK && (n < 0 || n > L)) {
            st = ORACLE_BAD_LEN;
        }
        double *K = NULL, *V = NULL, *qrow = NULL;
        if (st == ORACLE_OK) {
            K = malloc(sizeof(double) * ((size_t)L * D + 1));
            V = malloc(sizeof(double) * ((size_t)L * D + 1));
            qrow = malloc(sizeof(double) * (size_t)D);
            if (!K || !V || !qrow) {
                st = ORACLE_NO_MEMORY;
            } else {
                st = gather_context(pb, seq, kv_head, L, K, V);
            }
        }
        if (st == ORACLE_OK) {
            for (int32_t i = 0; i < n; ++i) {
                const int32_t visible = L - n + i + 1;      /* keys 0 .. L-n+i */
                for (int32_t hg = 0; hg < group; ++hg) {
                    const int32_t h = kv_head * group + hg;
                    const int64_t row = (int64_t)(q0 + i) * pb->num_q_heads + h;
                    for (int32_t d = 0; d < D; ++d) {
                        qrow[d] = widen(pb->q, row * D + d, q_dtype(pb));
                    }
                    double m, l;
                    attend_range(qrow, K, V, D, pb->scale, 0, visible, &m, &l, mp->out + row * D);
                }
            }
        } else {
            int expected = ORACLE_OK;
            __atomic_compare_exchange_n(&mp->status, &expected, st, 0, __ATOMIC_RELAXED,
                                        __ATOMIC_RELAXED);
        }
        free(K);
        free(V);
        free(qrow);
    }
    return NULL;
}

static int paged_multi_scaled(double *out, const void *q, const void *k_cache,
                              const void *v_cache, int32_t dtype, float k_scale, float v_scale,
                              const int32_t *block_tables, const int32_t *context_lens,
                              const int32_t *query_start_loc, int32_t num_seqs,
                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t block_size, int64_t num_blocks,
                              int32_t max_blocks_per_seq, float scale, int32_t num_threads);

/* out: [num_q_tokens][num_q_heads][head_dim] doubles, q: [num_q_tokens][Hq][D]. */
int oracle_paged_multi(double *out, const void *q, const void *k_cache, const void *v_cache,
                       int32_t dtype, const int32_t *block_tables, const int32_t *context_lens,
                       const int32_t *query_start_loc, int32_t num_seqs, int32_t num_q_heads,
                       int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                       int64_t num_blocks, int32_t max_blocks_per_seq, float scale,
                       int32_t num_threads)
{
    if (dtype != ORACLE_F32 && dtype != ORACLE_BF16) {
        return ORACLE_BAD_ARG;
    }
    return paged_multi_scaled(out, q, k_cache, v_cache, dtype, 1.0f, 1.0f, block_tables,
                              context_lens, query_start_loc, num_seqs, num_q_heads, num_kv_heads,
                              head_dim, block_size, num_blocks, max_blocks_per_seq, scale,
                              num_threads);
}

/* The same over FP8 (e4m3) pools: q is bf16; each cached element is its code's
 * value times k_scale (K pool) or v_scale (V pool). */
/* Decode over e5m2 pools (as oracle_paged_decode_fp8). */
int oracle_paged_decode_e5m2(double *out, const void *q, const void *k_cache,
                             const void *v_cache, float k_scale, float v_scale,
                             const int32_t *block_tables, const int32_t *context_lens,
                             int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                             int32_t head_dim, int32_t block_size, int64_t num_blocks,
                             int32_t max_blocks_per_seq, float scale,
                             const int32_t *tasks, int64_t num_tasks, int32_t num_threads)
{
    return paged_decode_scaled(out, q, k_cache, v_cache, ORACLE_E5M2, k_scale, v_scale,
                               block_tables, context_lens, num_seqs, num_q_heads, num_kv_heads,
                               head_dim, block_size, num_blocks, max_blocks_per_seq, scale,
                               tasks, num_tasks, num_threads);
}

int oracle_paged_multi_fp8(double *out, const void *q, const void *k_cache, const void *v_cache,
                           float k_scale, float v_scale, const int32_t *block_tables,
                           const int32_t *context_lens, const int32_t *query_start_loc,
                           int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size, int64_t num_blocks,
                           int32_t max_blocks_per_seq, float scale, int32_t num_threads)
{
    return paged_multi_scaled(out, q, k_cache, v_cache, ORACLE_E4M3, k_scale, v_scale,
                              block_tables, context_lens, query_start_loc, num_seqs, num_q_heads,
                              num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                              scale, num_threads);
}

/* Several query tokens over e5m2 pools. */
int oracle_paged_multi_e5m2(double *out, const void *q, const void *k_cache,
                            const void *v_cache, float k_scale, float v_scale,
                            const int32_t *block_tables, const int32_t *context_lens,
                            const int32_t *query_start_loc, int32_t num_seqs, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                            int64_t num_blocks, int32_t max_blocks_per_seq, float scale,
                            int32_t num_threads)
{
    return paged_multi_scaled(out, q, k_cache, v_cache, ORACLE_E5M2, k_scale, v_scale,
                              block_tables, context_lens, query_start_loc, num_seqs, num_q_heads,
                              num_kv_heads, head_dim, block_size, num_blocks, max_blocks_per_seq,
                              scale, num_threads);
}

static int paged_multi_scaled(double *out, const void *q, const void *k_cache,
                              const void *v_cache, int32_t dtype, float k_scale, float v_scale,
                              const int32_t *block_tables, const int32_t *context_lens,
                              const int32_t *query_start_loc, int32_t num_seqs,
                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t block_size, int64_t num_blocks,
                              int32_t max_blocks_per_seq, float scale, int32_t num_threads)
{
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens ||
        !query_start_loc || num_seqs < 0 ||
        num_q_heads <= 0 || num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 ||
        head_dim <= 0 || block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0) {
        return ORACLE_BAD_ARG;
    }
    for (int32_t s = 0; s < num_seqs; ++s) {
        if (query_start_loc[s + 1] < query_start_loc[s]) {
            return ORACLE_BAD_ARG;
        }
    }
    problem pb = {q, k_cache, v_cache, dtype, block_tables, context_lens,
                  num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                  num_blocks, max_blocks_per_seq, (double)scale, (double)k_scale,
                  (double)v_scale};
    multi_pool mp = {&pb, query_start_loc, out, 0, ORACLE_OK};
    if (num_threads <= 1) {
        multi_worker(&mp);
        return mp.status;
    }
    pthread_t *threads = malloc(sizeof(pthread_t) * (size_t)num_threads);
    if (!threads) {
        return ORACLE_NO_MEMORY;
    }
    int started = 0;
    for (int i = 0; i < num_threads; ++i) {
        if (pthread_create(&threads[i], NULL, multi_worker, &mp) != 0) {
            break;
        }
        ++started;
    }
    if (started == 0) {
        multi_worker(&mp);
    }
    for (int i = 0; i < started; ++i) {
        pthread_join(threads[i], NULL);
    }
    free(threads);
    return mp.status;
}

/* ------------------------------------------------------------------------- */
/* Partitioned attention and the log-sum-exp merge.
 *
 * The pages name online softmax only as a topic; the merge of partial softmax
 * results used here is the exact identity: with m_p the max score of part p,
 * l_p = sum exp(z - m_p) and o_p the part's normalised output,
 *   M = max_p m_p,  w_p = l_p exp(m_p - M),  out = sum_p w_p o_p / sum_p w_p,
 * which equals attention over the union of the parts.  Parts with l_p = 0
 * (empty) carry no weight. */

/* Statistics of the query (seq, q_head) over tokens [t0, t1). */
int oracle_partition_stats(const void *q, const void *k_cache, const void *v_cache,
                           int32_t dtype, const int32_t *block_tables,
                           const int32_t *context_lens, int32_t num_seqs,
                           int32_t num_q_heads, int32_t num_kv_heads,
                           int32_t head_dim, int32_t block_size, int64_t num_blocks,
                           int32_t max_blocks_per_seq, float scale, int32_t seq,
                           int32_t q_head, int32_t t0, int32_t t1, double *m,
                           double *l, double *o)
{
    if (!q || !k_cache || !v_cache || !block_tables || !context_lens || !m || !l ||
        !o || seq < 0 || seq >= num_seqs || q_head < 0 || q_head >= num_q_heads ||
        num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || t0 < 0 || t1 < t0) {
        return ORACLE_BAD_ARG;
    }
    problem pb = {q, k_cache, v_cache, dtype, block_tables, context_lens,
                  num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                  num_blocks, max_blocks_per_seq, (double)scale, 1.0, 1.0};
    int32_t L;
    int st = checked_len(&pb, seq, &L);
    if (st != ORACLE_OK) {
        return st;
    }
    if (t1 > L) {
        return ORACLE_BAD_ARG;
    }
    const int32_t D = head_dim;
    double *qrow = malloc(sizeof(double) * (size_t)D);
    double *K = malloc(sizeof(double) * ((size_t)L * D + 1));
    double *V = malloc(sizeof(double) * ((size_t)L * D + 1));
    if (!qrow || !K || !V) {
        free(qrow);
        free(K);
        free(V);
        return ORACLE_NO_MEMORY;
    }
    const int32_t kv_head = q_head / (num_q_heads / num_kv_heads);
    for (int32_t d = 0; d < D; ++d) {
        qrow[d] = widen(q, ((int64_t)seq * num_q_heads + q_head) * D + d,
                        is_fp8(dtype) ? ORACLE_BF16 : dtype);
    }
    st = gather_context(&pb, seq, kv_head, L, K, V);
    if (st == ORACLE_OK) {
        attend_range(qrow, K, V, D, (double)scale, t0, t1, m, l, o);
    }
    free(qrow);
    free(K);
    free(V);
    return st;
}

/* Merge nparts partial results (m[p], l[p], o[p*D .. p*D+D)) into out[0:D].
 * All parts empty gives a zero output. */
int oracle_lse_merge(const double *m, const double *l, const double *o,
                     int32_t nparts, int32_t head_dim, double *out)
{
    if (!m || !l || !o || !out || nparts < 0 || head_dim <= 0) {
        return ORACLE_BAD_ARG;
    }
    double M = -INFINITY;
    for (int32_t p = 0; p < nparts; ++p) {
        if (l[p] > 0.0 && m[p] > M) {
            M = m[p];
        }
    }
    for (int32_t d = 0; d < head_dim; ++d) {
        out[d] = 0.0;
    }
    if (M == -INFINITY) {
        return ORACLE_OK;
    }
    double total = 0.0;
    for (int32_t p = 0; p < nparts; ++p) {
        if (!(l[p] > 0.0)) {
            continue;
        }
        double w = l[p] * exp(m[p] - M);
        total += w;
        for (int32_t d = 0; d < head_dim; ++d) {
            out[d] += w * o[(int64_t)p * head_dim + d];
        }
    }
    for (int32_t d = 0; d < head_dim; ++d) {
        out[d] /= total;
    }
    return ORACLE_OK;
}

/* The same merge on single-precision partials (as a GPU writes them): each
 * value is widened to double, then merged as above. */
int oracle_lse_merge_f32(const float *m, const float *l, const float *o,
                         int32_t nparts, int32_t head_dim, double *out)
{
    if (!m || !l || !o || !out || nparts < 0 || head_dim <= 0) {
        return ORACLE_BAD_ARG;
    }
    double *md = malloc(sizeof(double) * (size_t)(nparts + 1));
    double *ld = malloc(sizeof(double) * (size_t)(nparts + 1));
    double *od = malloc(sizeof(double) * ((size_t)nparts * head_dim + 1));
    if (!md || !ld || !od) {
        free(md);
        free(ld);
        free(od);
        return ORACLE_NO_MEMORY;
    }
    for (int32_t p = 0; p < nparts; ++p) {
        md[p] = (double)m[p];
        ld[p] = (double)l[p];
        for (int32_t d = 0; d < head_dim; ++d) {
            od[(int64_t)p * head_dim + d] = (double)o[(int64_t)p * head_dim + d];
        }
    }
    int st = oracle_lse_merge(md, ld, od, nparts, head_dim, out);
    free(md);
    free(ld);
    free(od);
    return st;
}

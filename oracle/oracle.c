/*
 * Plain fp64 CPU oracle for the paged KV cache decode path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the benchmark's CPU
 * baseline leg do.  It shares no code, header or constant with the CUDA path.
 *
 * Every routine is the plain definition written out, in the order the pages
 * state it, with no blocking, fusion or reordering:
 *
 *   - The cache is split into fixed-size physical blocks of `block_size`
 *     tokens; a per-sequence block table maps logical block j to a physical
 *     block, and blocks may lie anywhere in the pool.
 *     ("PagedAttention: How vLLM Serves AI Like an Operating System",
 *      section "How It Works" and the "PagedAttention Memory Layout" example.)
 *   - Token position t (0-based) of a sequence sits in logical block
 *     t / block_size at offset t % block_size: the page's on-demand example
 *     opens a new block when the 17th and the 33rd token arrive.
 *     (same page, "The Magic: No Pre-allocation")
 *   - Attention over the paged cache equals ordinary softmax attention over
 *     the same tokens laid out contiguously: the paging is pure memory
 *     management and the method makes "no approximations".
 *     (same page, "Throughput Impact: The Numbers")
 *   - A block shared by several sequences is copied before it is modified
 *     (copy-on-write).  (same page, "Copy-on-Write: Sharing KV Cache")
 *
 * Cache layout (the pages give none; this is the layout both sides agree
 * on):  k_cache, v_cache : [num_blocks][num_kv_heads][block_size][head_dim],
 * row-major, elements of the input dtype.
 *
 * Precision: inputs are widened exactly to double; all arithmetic is fp64.
 * Writes and copies move element bytes unchanged.
 *
 * Element type codes used by this file only:  0 = fp32, 1 = fp16, 2 = bf16.
 *
 * Return codes: 0 = ok, -1 = invalid argument (the reason is in the
 * function's comment).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORC_F32 0
#define ORC_F16 1
#define ORC_BF16 2

static size_t elem_bytes(int dtype)
{
    return dtype == ORC_F32 ? 4u : 2u;
}

/* IEEE 754 binary16 -> double, from the format's definition:
 * 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits;
 * exponent 0 = zero/subnormal (fraction * 2^-24), exponent 31 = inf/NaN. */
static double half_bits_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double v;
    if (e == 0) {
        v = ldexp((double)f, -24);
    } else if (e == 31) {
        v = (f == 0) ? INFINITY : NAN;
    } else {
        v = ldexp((double)(f + 1024), e - 25);
    }
    return sign ? -v : v;
}

/* bfloat16 -> double: a bfloat16 is the upper 16 bits of an IEEE binary32. */
static double bf16_bits_to_double(uint16_t b)
{
    uint32_t u = (uint32_t)b << 16;
    float x;
    memcpy(&x, &u, sizeof x);
    return (double)x;
}

/* Element `idx` of an array of the given dtype, widened exactly. */
static double load_elem(const void* base, int64_t idx, int dtype)
{
    if (dtype == ORC_F32) {
        return (double)((const float*)base)[idx];
    }
    uint16_t bits = ((const uint16_t*)base)[idx];
    return dtype == ORC_F16 ? half_bits_to_double(bits) : bf16_bits_to_double(bits);
}

/* Exposed for the oracle's own self-test of the exact widening. */
double oracle_widen(const void* base, int64_t idx, int dtype)
{
    return load_elem(base, idx, dtype);
}

/*
 * Gather one sequence's keys and values for one kv head into contiguous fp64
 * arrays kc, vc of shape [ctx][head_dim]: token t comes from physical block
 * block_table[t / block_size], offset t % block_size.
 * ("How It Works": a block table maps logical to physical blocks;
 *  "The Magic: No Pre-allocation": the 17th token opens the second block.)
 * Returns -1 if a block id the sequence needs lies outside [0, num_blocks).
 */
int oracle_gather(double* kc, double* vc,
                  const void* k_cache, const void* v_cache,
                  const int32_t* block_table, int32_t ctx,
                  int32_t kv_head, int32_t num_kv_heads, int32_t head_dim,
                  int32_t block_size, int32_t num_blocks, int dtype)
{
    for (int32_t t = 0; t < ctx; ++t) {
        int32_t logical = t / block_size;
        int32_t offset = t % block_size;
        int32_t phys = block_table[logical];
        if (phys < 0 || phys >= num_blocks) {
            return -1;
        }
        int64_t row = (((int64_t)phys * num_kv_heads + kv_head) * block_size + offset) * head_dim;
        for (int32_t d = 0; d < head_dim; ++d) {
            kc[(int64_t)t * head_dim + d] = load_elem(k_cache, row + d, dtype);
            vc[(int64_t)t * head_dim + d] = load_elem(v_cache, row + d, dtype);
        }
    }
    return 0;
}

/*
 * Textbook softmax attention of one query vector q[head_dim] over ctx
 * contiguous keys/values (fp64):
 *     s_t = scale * sum_d q[d] * K[t][d]
 *     p_t = exp(s_t - max_u s_u) / sum_u exp(s_u - max_u s_u)
 *     out[d] = sum_t p_t * V[t][d]
 * Two passes over the scores (max, then exponentials); no causal mask, as
 * the single decode query attends to every cached token.
 * `scores` is caller scratch of ctx doubles.  ctx must be >= 1.
 */
static void attend_contiguous(double* out, const double* q, const double* kc,
                              const double* vc, int32_t ctx, int32_t head_dim,
                              double scale, double* scores)
{
    double smax = -INFINITY;
    for (int32_t t = 0; t < ctx; ++t) {
        double dot = 0.0;
        for (int32_t d = 0; d < head_dim; ++d) {
            dot += q[d] * kc[(int64_t)t * head_dim + d];
        }
        scores[t] = scale * dot;
        if (scores[t] > smax) {
            smax = scores[t];
        }
    }
    double denom = 0.0;
    for (int32_t t = 0; t < ctx; ++t) {
        scores[t] = exp(scores[t] - smax);
        denom += scores[t];
    }
    for (int32_t d = 0; d < head_dim; ++d) {
        out[d] = 0.0;
    }
    for (int32_t t = 0; t < ctx; ++t) {
        double p = scores[t] / denom;
        for (int32_t d = 0; d < head_dim; ++d) {
            out[d] += p * vc[(int64_t)t * head_dim + d];
        }
    }
}

/*
 * Decode attention for ONE sequence s, all its query heads:
 *   out[i][d] for i in [0, num_q_heads), written to out_seq[num_q_heads][head_dim].
 * Query head i reads kv head i / (num_q_heads / num_kv_heads) (consecutive
 * grouping of query heads onto shared kv heads).
 * q_seq points at this sequence's queries [num_q_heads][head_dim];
 * block_table at this sequence's row; ctx = its context length (>= 1).
 * Returns -1 on ctx < 1, ctx beyond the row, a bad head split or a bad id.
 */
int oracle_paged_decode_seq(double* out_seq, const void* q_seq,
                            const void* k_cache, const void* v_cache,
                            const int32_t* block_table, int32_t max_blocks_per_seq,
                            int32_t ctx, int32_t num_q_heads, int32_t num_kv_heads,
                            int32_t head_dim, int32_t block_size, int32_t num_blocks,
                            double scale, int dtype)
{
    if (ctx < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads != 0 || block_size < 1 ||
        (int64_t)ctx > (int64_t)max_blocks_per_seq * block_size) {
        return -1;
    }
    int32_t group = num_q_heads / num_kv_heads;
    double* kc = (double*)malloc(sizeof(double) * (size_t)ctx * head_dim);
    double* vc = (double*)malloc(sizeof(double) * (size_t)ctx * head_dim);
    double* scores = (double*)malloc(sizeof(double) * (size_t)ctx);
    double* qd = (double*)malloc(sizeof(double) * (size_t)head_dim);
    int rc = (kc && vc && scores && qd) ? 0 : -1;
    for (int32_t h = 0; rc == 0 && h < num_kv_heads; ++h) {
        rc = oracle_gather(kc, vc, k_cache, v_cache, block_table, ctx, h, num_kv_heads,
                           head_dim, block_size, num_blocks, dtype);
        for (int32_t i = h * group; rc == 0 && i < (h + 1) * group; ++i) {
            for (int32_t d = 0; d < head_dim; ++d) {
                qd[d] = load_elem(q_seq, (int64_t)i * head_dim + d, dtype);
            }
            attend_contiguous(out_seq + (int64_t)i * head_dim, qd, kc, vc, ctx, head_dim,
                              scale, scores);
        }
    }
    free(kc);
    free(vc);
    free(scores);
    free(qd);
    return rc;
}

/*
 * Decode attention for a whole batch: out[num_seqs][num_q_heads][head_dim]
 * (fp64), q[num_seqs][num_q_heads][head_dim], block_tables
 * [num_seqs][max_blocks_per_seq], context_lens[num_seqs].
 */
int oracle_paged_decode(double* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq,
                        const int32_t* context_lens, int32_t num_seqs, int32_t num_q_heads,
                        int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                        int32_t num_blocks, double scale, int dtype)
{
    size_t eb = elem_bytes(dtype);
    for (int32_t s = 0; s < num_seqs; ++s) {
        const char* q_seq = (const char*)q + (size_t)s * num_q_heads * head_dim * eb;
        int rc = oracle_paged_decode_seq(out + (int64_t)s * num_q_heads * head_dim, q_seq,
                                         k_cache, v_cache,
                                         block_tables + (int64_t)s * max_blocks_per_seq,
                                         max_blocks_per_seq, context_lens[s], num_q_heads,
                                         num_kv_heads, head_dim, block_size, num_blocks,
                                         scale, dtype);
        if (rc != 0) {
            return rc;
        }
    }
    return 0;
}

/*
 * Multi-query decode: each sequence brings q_len new tokens (for example
 * draft tokens to verify), already counted in context_lens.  New token j
 * (0-based) sits at position ctx - q_len + j and, as in any causal decoder,
 * attends to every token up to and including its own position, i.e. to the
 * first ctx - q_len + j + 1 tokens.  q and out are
 * [num_seqs][q_len][num_q_heads][head_dim].  With q_len = 1 this is
 * oracle_paged_decode.  (Speculative decoding, "PagedAttention & Continuous
 * Batching: How vLLM Achieves 24x Serving Throughput", item 7: the target
 * model checks several proposed tokens in one pass.)
 * Returns -1 if some ctx < q_len or on any error of the single-query form.
 */
int oracle_paged_decode_mq(double* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t num_seqs, int32_t q_len,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int32_t num_blocks, double scale, int dtype)
{
    size_t eb = elem_bytes(dtype);
    if (q_len < 1) {
        return -1;
    }
    for (int32_t s = 0; s < num_seqs; ++s) {
        int32_t ctx = context_lens[s];
        if (ctx < q_len) {
            return -1;
        }
        for (int32_t j = 0; j < q_len; ++j) {
            int64_t row = (int64_t)s * q_len + j;
            const char* q_row = (const char*)q + (size_t)row * num_q_heads * head_dim * eb;
            int rc = oracle_paged_decode_seq(out + row * num_q_heads * head_dim, q_row, k_cache,
                                             v_cache, block_tables + (int64_t)s * max_blocks_per_seq,
                                             max_blocks_per_seq, ctx - q_len + j + 1, num_q_heads,
                                             num_kv_heads, head_dim, block_size, num_blocks, scale,
                                             dtype);
            if (rc != 0) {
                return rc;
            }
        }
    }
    return 0;
}

/*
 * Slot write: for token t with slot = slot_mapping[t] >= 0, store its key and
 * value rows (every kv head) at physical block slot / block_size, offset
 * slot % block_size.  A negative slot means "no write" (padding token).
 * Element bytes are copied unchanged.
 * ("How It Works": blocks are filled only when new tokens need storing.)
 * Returns -1 (before writing anything) if a slot lies beyond the pool.
 */
int oracle_kv_write(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                    const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                    int32_t head_dim, int32_t block_size, int32_t num_blocks, int dtype)
{
    size_t eb = elem_bytes(dtype);
    size_t row_bytes = (size_t)head_dim * eb;
    for (int32_t t = 0; t < num_tokens; ++t) {
        if (slot_mapping[t] >= (int64_t)num_blocks * block_size) {
            return -1;
        }
    }
    for (int32_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) {
            continue;
        }
        int64_t blk = slot / block_size;
        int64_t off = slot % block_size;
        for (int32_t h = 0; h < num_kv_heads; ++h) {
            size_t dst = (size_t)(((blk * num_kv_heads + h) * block_size + off) * head_dim) * eb;
            size_t src = (size_t)(((int64_t)t * num_kv_heads + h) * head_dim) * eb;
            memcpy((char*)k_cache + dst, (const char*)k_new + src, row_bytes);
            memcpy((char*)v_cache + dst, (const char*)v_new + src, row_bytes);
        }
    }
    return 0;
}

/*
 * Copy-on-write block copy: for each pair (src, dst), in the order given,
 * the whole physical block dst (keys and values, every kv head) becomes a
 * copy of block src.  ("Copy-on-Write: Sharing KV Cache": a request that
 * must modify a shared block copies it first.)
 * pairs = [n][2] int64 as (src, dst).  Returns -1 (before copying) for an id
 * outside the pool, src == dst, a dst named twice, or a dst that is also a
 * src of this call -- in those cases the result would depend on the order.
 */
int oracle_block_copy(void* k_cache, void* v_cache, const int64_t* pairs, int32_t n,
                      int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                      int32_t num_blocks, int dtype)
{
    for (int32_t i = 0; i < n; ++i) {
        int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks || src == dst) {
            return -1;
        }
        for (int32_t j = 0; j < n; ++j) {
            if (j != i && pairs[2 * j + 1] == dst) {
                return -1;
            }
            if (pairs[2 * j] == dst) {
                return -1;
            }
        }
    }
    size_t block_bytes = (size_t)num_kv_heads * block_size * head_dim * elem_bytes(dtype);
    for (int32_t i = 0; i < n; ++i) {
        int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        memcpy((char*)k_cache + (size_t)dst * block_bytes,
               (const char*)k_cache + (size_t)src * block_bytes, block_bytes);
        memcpy((char*)v_cache + (size_t)dst * block_bytes,
               (const char*)v_cache + (size_t)src * block_bytes, block_bytes);
    }
    return 0;
}

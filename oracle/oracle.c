/*
 * oracle.c -- slow, plain, double-precision CPU oracle for paged attention
 * over a block-table KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is compiled into its own shared
 * library and is called only by the test suite, by the smoke check and by
 * the CPU-baseline leg of the benchmark.  It shares no code, header or
 * constant with the CUDA library and never calls it.
 *
 * What it computes follows the pages this project is built from:
 *   [P1] "tiny-vllm：从零构建高性能LLM推理引擎的完整指南" (zingnex.cn)
 *        sec. "PagedAttention：从操作系统借来的智慧": the KV cache is cut into
 *          fixed-size blocks; a per-sequence block table maps logical blocks
 *          to (non-contiguous) physical blocks.
 *        sec. "Llama 3.2 1B架构拆解": grouped-query attention (fewer KV heads
 *          than query heads), causal mask, softmax, weighted sum of V.
 *        sec. "推理流程：从Prefill到Decode": decode computes the new token's
 *          K,V and appends them to the cache, then attends over the cache.
 *        sec. "在线Softmax": numerically stable softmax (running max).
 *        sec. "BF16浮点数": bf16 = 1 sign, 8 exponent, 7 mantissa bits,
 *          i.e. the top 16 bits of an IEEE-754 binary32.
 *   [P3] "Tiny-vLLM 实战：用 C++/CUDA 手写高性能 LLM 推理引擎" (hotdry.top)
 *        sec. "内存池管理": a page holds page_size x head_dim x num_kv_heads
 *          bf16 values (16 x 512 x 2 B = 16 KB for Llama-3.2-1B).
 *
 * Readings where the pages are silent (each one is listed in the design
 * notes of the repository):
 *   - pool layout [num_pages][page_size][num_kv_heads][head_dim], one pool
 *     for K and one for V;
 *   - query head h reads KV head h / (num_q_heads / num_kv_heads);
 *   - slot = page * page_size + offset; a negative slot is padding;
 *   - context_lens counts the tokens after the append, so a decode query sits
 *     at position context_len - 1 and sees keys 0 .. context_len - 1;
 *   - chunked prefill: the chunk's K,V are appended first; query i of a chunk
 *     of T tokens over context C sits at position C - T + i and sees keys
 *     0 .. C - T + i;
 *   - split partitions are logical token ranges [p*PT, (p+1)*PT) from 0,
 *     each with its own normalised output and natural-log sum-exp;
 *   - an empty key range gives output 0 and log-sum-exp -infinity.
 *
 * The arithmetic is the plain definition: every bf16 decoded exactly to a
 * double, scores s_j = scale * <q, K_j>, a first pass for m = max_j s_j, a
 * second for w_j = exp(s_j - m), l = sum w_j, out = sum w_j V_j / l.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* [P1] sec. "BF16浮点数": a bf16 value is the upper half of a binary32. */
static double bf16_value(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Physical row of logical token j of one sequence, through its block table
 * ([P1] sec. "PagedAttention"): block j / PS, offset j % PS.  Returns a
 * pointer to the [num_kv_heads][head_dim] row, or NULL when the table entry
 * is outside the pool. */
static const uint16_t *token_row(const uint16_t *pool, const int32_t *bt_row,
                                 int64_t j, int page_size, int64_t num_pages,
                                 int row_elems)
{
    int64_t logical_block = j / page_size;
    int64_t offset = j % page_size;
    int64_t page = bt_row[logical_block];
    if (page < 0 || page >= num_pages)
        return NULL;
    return pool + (page * page_size + offset) * (int64_t)row_elems;
}

/* Attention of one query row q[0..D) of KV head g over keys [j0, j1) of one
 * sequence.  Writes out[0..D) and *lse (natural log of sum exp of scaled
 * scores).  Returns the number of keys whose page id was out of range (those
 * keys are left out). */
static int attend(const uint16_t *q, const uint16_t *k_pool,
                  const uint16_t *v_pool, const int32_t *bt_row,
                  int64_t j0, int64_t j1, int g, int num_kv_heads,
                  int head_dim, int page_size, int64_t num_pages,
                  double scale, double *out, double *lse)
{
    int row_elems = num_kv_heads * head_dim;
    int bad = 0;
    for (int d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    *lse = -INFINITY;
    if (j1 <= j0)
        return 0;

    int64_t n = j1 - j0;
    double *s = (double *)malloc((size_t)n * sizeof(double));
    unsigned char *ok = (unsigned char *)malloc((size_t)n);

    /* pass 1: scores and their maximum */
    double m = -INFINITY;
    for (int64_t j = j0; j < j1; ++j) {
        const uint16_t *krow = token_row(k_pool, bt_row, j, page_size,
                                         num_pages, row_elems);
        ok[j - j0] = krow != NULL;
        if (!krow) {
            ++bad;
            continue;
        }
        krow += (int64_t)g * head_dim;
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d)
            dot += bf16_value(q[d]) * bf16_value(krow[d]);
        s[j - j0] = scale * dot;
        if (s[j - j0] > m)
            m = s[j - j0];
    }

    /* pass 2: exponentials, their sum and the weighted sum of V */
    double l = 0.0;
    for (int64_t j = j0; j < j1; ++j) {
        if (!ok[j - j0])
            continue;
        const uint16_t *vrow = token_row(v_pool, bt_row, j, page_size,
                                         num_pages, row_elems);
        vrow += (int64_t)g * head_dim;
        double w = exp(s[j - j0] - m);
        l += w;
        for (int d = 0; d < head_dim; ++d)
            out[d] += w * bf16_value(vrow[d]);
    }
    if (l > 0.0) {
        for (int d = 0; d < head_dim; ++d)
            out[d] /= l;
        *lse = m + log(l);
    }
    free(s);
    free(ok);
    return bad;
}

/*
 * RoPE on K rows ([P1] sec. "Llama 3.2 1B架构拆解": rotary position encoding
 * injects the position into Q and K by rotation).  The pages give neither
 * the pairing of dimensions nor the angles nor the arithmetic; the readings:
 *   - dimension i is rotated together with i + head_dim/2 (the rotate-half
 *     convention of the Hugging Face Llama model the pages dump);
 *   - the angles come from a caller table cos_sin[position][2][head_dim/2]
 *     (the cos row, then the sin row), so any frequency base or scaling is
 *     the caller's;
 *   - the arithmetic is binary32: with x1 = k[i], x2 = k[i + D/2],
 *       y1 = fl(fl(x1 * c) - fl(x2 * s)),  y2 = fl(fl(x2 * c) + fl(x1 * s)),
 *     fl() rounding to nearest binary32 (no fused multiply-add), and the
 *     result is rounded to bf16 (nearest even) as it enters the pool.
 * A row whose position is outside [0, max_position) is left unrotated and
 * counted.
 */
static uint16_t bf16_round_nearest_even(float f)
{
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu))
        return (uint16_t)((u >> 16) | 0x40u);          /* quiet NaN */
    u += 0x7fffu + ((u >> 16) & 1u);
    return (uint16_t)(u >> 16);
}

int64_t oracle_rope_rows(uint16_t *rows, const int32_t *positions,
                         int64_t num_rows, int num_kv_heads, int head_dim,
                         const float *cos_sin, int max_position)
{
    const int half = head_dim / 2;
    int64_t bad = 0;
    for (int64_t t = 0; t < num_rows; ++t) {
        const int pos = positions[t];
        if (pos < 0 || pos >= max_position) {
            ++bad;
            continue;
        }
        const float *cs = cos_sin + (int64_t)pos * head_dim;
        for (int h = 0; h < num_kv_heads; ++h) {
            uint16_t *k = rows + (t * num_kv_heads + h) * (int64_t)head_dim;
            for (int i = 0; i < half; ++i) {
                const float x1 = (float)bf16_value(k[i]);
                const float x2 = (float)bf16_value(k[i + half]);
                const float c = cs[i], s = cs[half + i];
                const float a = x1 * c, b = x2 * s;
                const float e = x2 * c, f = x1 * s;
                const float y1 = a - b, y2 = e + f;
                k[i] = bf16_round_nearest_even(y1);
                k[i + half] = bf16_round_nearest_even(y2);
            }
        }
    }
    return bad;
}

void oracle_set_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* KV append ([P1] sec. "推理流程"; [P3] sec. "内存池管理"): token t's K row
 * and V row ([num_kv_heads][head_dim] bf16) are copied into slot
 * slot_mapping[t] of the pools.  Negative slots are skipped.  Returns the
 * number of tokens whose slot lies beyond the pool (those are skipped too). */
int64_t oracle_kv_append(const uint16_t *k_new, const uint16_t *v_new,
                         const int32_t *slot_mapping, int64_t num_tokens,
                         uint16_t *k_pool, uint16_t *v_pool,
                         int64_t num_pages, int num_kv_heads, int head_dim,
                         int page_size)
{
    int64_t row_elems = (int64_t)num_kv_heads * head_dim;
    int64_t num_slots = num_pages * page_size;
    int64_t bad = 0;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= num_slots) {
            ++bad;
            continue;
        }
        int64_t page = slot / page_size;
        int64_t offset = slot % page_size;
        int64_t dst = (page * page_size + offset) * row_elems;
        memcpy(k_pool + dst, k_new + t * row_elems, (size_t)row_elems * 2);
        memcpy(v_pool + dst, v_new + t * row_elems, (size_t)row_elems * 2);
    }
    return bad;
}

/* Decode ([P1] secs. "推理流程", "PagedAttention", "Llama 3.2 1B架构拆解"):
 * one query per sequence at position context_lens[s] - 1, attending to keys
 * 0 .. context_lens[s] - 1.  Rows (seq_idx[r], head_idx[r]) for r < nrows
 * are computed; out is [nrows][head_dim].  Returns the count of keys left
 * out because of a bad page id. */
int64_t oracle_paged_decode_rows(double *out, double *lse,
                                 const int32_t *seq_idx,
                                 const int32_t *head_idx, int64_t nrows,
                                 const uint16_t *q, const uint16_t *k_pool,
                                 const uint16_t *v_pool,
                                 const int32_t *block_tables,
                                 int max_blocks_per_seq,
                                 const int32_t *context_lens, int num_q_heads,
                                 int num_kv_heads, int head_dim,
                                 int page_size, int64_t num_pages,
                                 double scale)
{
    int group = num_q_heads / num_kv_heads;
    int64_t bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(+ : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t s = seq_idx[r];
        int h = head_idx[r];
        double row_lse;
        bad += attend(q + (s * num_q_heads + h) * (int64_t)head_dim, k_pool,
                      v_pool, block_tables + s * (int64_t)max_blocks_per_seq,
                      0, context_lens[s], h / group, num_kv_heads, head_dim,
                      page_size, num_pages, scale, out + r * head_dim,
                      &row_lse);
        if (lse)
            lse[r] = row_lse;
    }
    return bad;
}

/* Split-KV partials (blockwise form of [P1] sec. "在线Softmax", and of the
 * tiled attention of [P3] sec. "算子融合"): partition p of sequence s covers
 * logical keys [p*PT, min((p+1)*PT, context_len)).  For every (s, h, p <
 * max_partitions): o_p[s][h][p][:] is the normalised attention over that
 * range and lse_p[s][h][p] its natural log-sum-exp (-inf when empty). */
int64_t oracle_paged_decode_partials(double *o_p, double *lse_p,
                                     const uint16_t *q,
                                     const uint16_t *k_pool,
                                     const uint16_t *v_pool,
                                     const int32_t *block_tables,
                                     int max_blocks_per_seq,
                                     const int32_t *context_lens,
                                     int num_seqs, int num_q_heads,
                                     int num_kv_heads, int head_dim,
                                     int page_size, int64_t num_pages,
                                     double scale, int partition_tokens,
                                     int max_partitions)
{
    int group = num_q_heads / num_kv_heads;
    int64_t total = (int64_t)num_seqs * num_q_heads * max_partitions;
    int64_t bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(+ : bad)
    for (int64_t idx = 0; idx < total; ++idx) {
        int64_t p = idx % max_partitions;
        int64_t sh = idx / max_partitions;
        int h = (int)(sh % num_q_heads);
        int64_t s = sh / num_q_heads;
        int64_t ctx = context_lens[s];
        int64_t j0 = p * (int64_t)partition_tokens;
        int64_t j1 = j0 + partition_tokens;
        if (j1 > ctx)
            j1 = ctx;
        bad += attend(q + (s * num_q_heads + h) * (int64_t)head_dim, k_pool,
                      v_pool, block_tables + s * (int64_t)max_blocks_per_seq,
                      j0, j1, h / group, num_kv_heads, head_dim, page_size,
                      num_pages, scale, o_p + idx * head_dim, lse_p + idx);
    }
    return bad;
}

/* Log-sum-exp merge of split partials: with M = max_p lse_p over the
 * non-empty partitions p < ceil(context_len / PT),
 *   out = sum_p exp(lse_p - M) o_p / sum_p exp(lse_p - M).
 * A sequence with no keys gets out = 0. */
void oracle_split_merge(double *out, const double *o_p, const double *lse_p,
                        const int32_t *context_lens, int num_seqs,
                        int num_q_heads, int head_dim, int partition_tokens,
                        int max_partitions)
{
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t ctx = context_lens[s];
        int64_t nparts = (ctx + partition_tokens - 1) / partition_tokens;
        if (nparts > max_partitions)
            nparts = max_partitions;
        for (int h = 0; h < num_q_heads; ++h) {
            int64_t base = (s * num_q_heads + h) * (int64_t)max_partitions;
            double *o = out + (s * num_q_heads + h) * (int64_t)head_dim;
            for (int d = 0; d < head_dim; ++d)
                o[d] = 0.0;
            double m = -INFINITY;
            for (int64_t p = 0; p < nparts; ++p)
                if (lse_p[base + p] > m)
                    m = lse_p[base + p];
            if (m == -INFINITY)
                continue;
            double wsum = 0.0;
            for (int64_t p = 0; p < nparts; ++p) {
                if (lse_p[base + p] == -INFINITY)
                    continue;
                double w = exp(lse_p[base + p] - m);
                wsum += w;
                for (int d = 0; d < head_dim; ++d)
                    o[d] += w * o_p[(base + p) * head_dim + d];
            }
            for (int d = 0; d < head_dim; ++d)
                o[d] /= wsum;
        }
    }
}

/* Chunked prefill ([P1] sec. "推理流程": prefill handles all prompt tokens
 * at once under a causal mask).  Sequence s owns query rows
 * [query_start_loc[s], query_start_loc[s+1]) of q ([rows][Hq][D]); with
 * T = that count and C = context_lens[s], row i sits at position C - T + i
 * and attends to keys 0 .. C - T + i.  Rows (tok_idx[r], head_idx[r]) are
 * computed into out[r][:]. */
int64_t oracle_paged_prefill_rows(double *out, const int32_t *tok_idx,
                                  const int32_t *head_idx, int64_t nrows,
                                  const uint16_t *q,
                                  const int32_t *query_start_loc,
                                  const uint16_t *k_pool,
                                  const uint16_t *v_pool,
                                  const int32_t *block_tables,
                                  int max_blocks_per_seq,
                                  const int32_t *context_lens, int num_seqs,
                                  int num_q_heads, int num_kv_heads,
                                  int head_dim, int page_size,
                                  int64_t num_pages, double scale)
{
    int group = num_q_heads / num_kv_heads;
    int64_t bad = 0;
#pragma omp parallel for schedule(dynamic) reduction(+ : bad)
    for (int64_t r = 0; r < nrows; ++r) {
        int64_t t = tok_idx[r];
        int h = head_idx[r];
        int64_t s = 0;
        while (s + 1 < num_seqs && query_start_loc[s + 1] <= t)
            ++s;
        int64_t chunk = query_start_loc[s + 1] - query_start_loc[s];
        int64_t i = t - query_start_loc[s];
        int64_t pos = context_lens[s] - chunk + i;
        double row_lse;
        bad += attend(q + (t * num_q_heads + h) * (int64_t)head_dim, k_pool,
                      v_pool, block_tables + s * (int64_t)max_blocks_per_seq,
                      0, pos + 1, h / group, num_kv_heads, head_dim,
                      page_size, num_pages, scale, out + r * head_dim,
                      &row_lse);
    }
    return bad;
}

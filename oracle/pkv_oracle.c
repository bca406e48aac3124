/*
 * pkv_oracle.c -- plain, slow, fp64 CPU oracle for paged-KV decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, import or
 * call this file: only the tests, the smoke check and the benchmark's CPU
 * baseline leg use it.  It shares no code, header, constant or helper with the
 * CUDA library; it decodes fp16/bf16 bits itself and gathers every key/value
 * through the block table one position at a time.
 *
 * What it computes, and where that is stated:
 *
 *   - KV append: "the cache stores K and V for every past position and appends
 *     the new token's K and V each step" -- page "LLM Inference: KV Cache,
 *     Batching & Scheduling" (cariara.com), section "The KV cache".
 *     oracle_append() is the byte copy cache[slot] <- new for every slot >= 0.
 *
 *   - Paged storage: KV lives in fixed-size blocks (typically 16 tokens; 16 or
 *     32 in the other two pages); a per-sequence table maps logical blocks to
 *     physical ones like OS virtual memory -- same page, section
 *     "PagedAttention and vLLM"; and page "LLM Inference Engineering:
 *     Overcoming the KV-Cache Bottleneck..." (wpnews.pro summary), section
 *     "2. The Architectural Solution: Virtual Memory and PagedAttention".
 *     Position p of a sequence lives in physical block table[p / bs] at row
 *     p % bs.
 *
 *   - Attention over the cached context: "Attention needs the keys and values
 *     of all prior positions" (cariara.com page, section "The KV cache").  The
 *     oracle evaluates the plain definition
 *         z[p]  = scale * sum_d q[d] * K[p][d]
 *         m     = max_p z[p],  w[p] = exp(z[p] - m),  L = sum_p w[p]
 *         out   = sum_p (w[p] / L) * V[p]
 *     in fp64, two passes, no online rescaling.  Query head h reads KV head
 *     h / G with G = Hq / Hkv (contiguous query-head groups share one KV head;
 *     the page names "KV heads (GQA)" in the same section).
 *
 *   - Partitioned context + log-sum-exp merge: not on the pages.  The identity
 *     softmax(z)V = sum_j exp(m_j - M) o_j / sum_j exp(m_j - M) l_j over any
 *     partition of the positions is exact mathematics; oracle_attention_range()
 *     and oracle_lse_merge() state it so a test can check it in fp64.
 *
 *   - KV sizing: "2 * seq_len * num_heads * head_dim * sizeof(dtype)" bytes per
 *     layer, with num_heads the KV heads in the worked table (cariara.com page,
 *     section "The KV cache").
 *
 * Layouts (the library's documented ABI, restated here independently):
 *   q            [B][Hq][D]        16-bit floats (dtype 0 = IEEE fp16, 1 = bf16)
 *   k/v cache    [NB][Hkv][bs][D]  16-bit floats
 *   block_tables [B][MB]           int32 physical block ids
 *   context_lens [B]               int32, positions 0..ctx-1 are attended
 *   out          [npairs][D]       fp64
 *
 * A context length of 0 yields an all-zero output row (no positions).
 * Return codes: 0 ok, -1 invalid argument / table entry out of range.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ---- 16-bit float decoding, written from the IEEE-754 binary16 and the
 *      bfloat16 (upper half of binary32) definitions. ---------------------- */

double oracle_half_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int exp = (h >> 10) & 0x1f;
    int man = h & 0x3ff;
    double v;
    if (exp == 0) {
        v = ldexp((double)man, -24);               /* subnormal: man * 2^-24 */
    } else if (exp == 31) {
        v = man ? NAN : INFINITY;
    } else {
        v = ldexp((double)(man | 0x400), exp - 25); /* (1.man) * 2^(exp-15) */
    }
    return sign ? -v : v;
}

double oracle_bf16_to_double(uint16_t b)
{
    uint32_t bits = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static double decode16(int dtype, uint16_t x)
{
    return dtype == 0 ? oracle_half_to_double(x) : oracle_bf16_to_double(x);
}

/* ---- sizing (cariara.com page, "The KV cache": per-layer memory cost) ----- */

int64_t oracle_kv_bytes_per_layer(int64_t seq_len, int64_t kv_heads,
                                  int64_t head_dim, int64_t dtype_bytes)
{
    /* one K and one V vector per head per position */
    return 2 * seq_len * kv_heads * head_dim * dtype_bytes;
}

/* ---- paging address: position p -> flat slot (block * bs + row) ---------- */

int64_t oracle_slot_of(const int32_t *table_row, int64_t pos, int64_t block_size)
{
    int64_t logical_block = pos / block_size;
    int64_t row = pos % block_size;
    return (int64_t)table_row[logical_block] * block_size + row;
}

/* ---- append: cache[slot] <- new for each token with slot >= 0 ------------ */

int oracle_append(uint16_t *cache, int64_t num_blocks, int64_t kv_heads,
                  int64_t block_size, int64_t head_dim,
                  const uint16_t *new_kv, const int64_t *slot_mapping,
                  int64_t num_tokens)
{
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;                               /* padding token: no write */
        int64_t block = slot / block_size;
        int64_t row = slot % block_size;
        if (block >= num_blocks)
            return -1;
        for (int64_t h = 0; h < kv_heads; ++h) {
            uint16_t *dst = cache + ((block * kv_heads + h) * block_size + row) * head_dim;
            const uint16_t *src = new_kv + (t * kv_heads + h) * head_dim;
            memcpy(dst, src, (size_t)head_dim * sizeof(uint16_t));
        }
    }
    return 0;
}

/* ---- gather one position's K or V row for KV head g ---------------------- */

static int gather_row(const uint16_t *cache, int dtype, int64_t num_blocks,
                      int64_t kv_heads, int64_t block_size, int64_t head_dim,
                      const int32_t *table_row, int64_t pos, int64_t g,
                      double *dst)
{
    int64_t block = table_row[pos / block_size];
    int64_t row = pos % block_size;
    if (block < 0 || block >= num_blocks)
        return -1;
    const uint16_t *src = cache + ((block * kv_heads + g) * block_size + row) * head_dim;
    for (int64_t d = 0; d < head_dim; ++d)
        dst[d] = decode16(dtype, src[d]);
    return 0;
}

/*
 * Unnormalised attention of one (sequence, query head) over positions
 * [p_begin, p_end):  m = max z (natural-log domain), l = sum exp(z - m),
 * o[d] = sum exp(z - m) V[d].  An empty range gives m = -inf, l = 0, o = 0.
 */
int oracle_attention_range(int dtype, const uint16_t *q, int64_t num_q_heads,
                           const uint16_t *k_cache, const uint16_t *v_cache,
                           int64_t num_blocks, int64_t block_size,
                           int64_t num_kv_heads, int64_t head_dim,
                           const int32_t *block_tables, int64_t max_blocks_per_seq,
                           double scale, int64_t seq, int64_t head,
                           int64_t p_begin, int64_t p_end,
                           double *m_out, double *l_out, double *o_out)
{
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
        return -1;
    if (p_end > max_blocks_per_seq * block_size || p_begin < 0)
        return -1;
    int64_t group = num_q_heads / num_kv_heads;
    int64_t g = head / group;
    const int32_t *table_row = block_tables + seq * max_blocks_per_seq;
    const uint16_t *qh = q + (seq * num_q_heads + head) * head_dim;
    int64_t n = p_end > p_begin ? p_end - p_begin : 0;

    for (int64_t d = 0; d < head_dim; ++d)
        o_out[d] = 0.0;
    if (n == 0) {
        *m_out = -INFINITY;
        *l_out = 0.0;
        return 0;
    }

    double *qd = malloc(sizeof(double) * head_dim);
    double *row = malloc(sizeof(double) * head_dim);
    double *z = malloc(sizeof(double) * n);
    int rc = 0;
    if (!qd || !row || !z) {
        rc = -1;
        goto done;
    }
    for (int64_t d = 0; d < head_dim; ++d)
        qd[d] = decode16(dtype, qh[d]);

    /* pass 1: scores */
    double m = -INFINITY;
    for (int64_t i = 0; i < n; ++i) {
        if (gather_row(k_cache, dtype, num_blocks, num_kv_heads, block_size,
                       head_dim, table_row, p_begin + i, g, row)) {
            rc = -1;
            goto done;
        }
        double dot = 0.0;
        for (int64_t d = 0; d < head_dim; ++d)
            dot += qd[d] * row[d];
        z[i] = scale * dot;
        if (z[i] > m)
            m = z[i];
    }
    /* pass 2: weights and weighted value sum */
    double l = 0.0;
    for (int64_t i = 0; i < n; ++i) {
        double w = exp(z[i] - m);
        l += w;
        if (gather_row(v_cache, dtype, num_blocks, num_kv_heads, block_size,
                       head_dim, table_row, p_begin + i, g, row)) {
            rc = -1;
            goto done;
        }
        for (int64_t d = 0; d < head_dim; ++d)
            o_out[d] += w * row[d];
    }
    *m_out = m;
    *l_out = l;
done:
    free(qd);
    free(row);
    free(z);
    return rc;
}

/*
 * Full decode attention for a list of (sequence, query head) pairs, or for
 * all B * Hq pairs when pairs == NULL.  out is [npairs][D] fp64:
 * out = o / l over positions [0, ctx).
 */
int oracle_paged_attention(int dtype, const uint16_t *q, int64_t num_seqs,
                           int64_t num_q_heads, const uint16_t *k_cache,
                           const uint16_t *v_cache, int64_t num_blocks,
                           int64_t block_size, int64_t num_kv_heads,
                           int64_t head_dim, const int32_t *block_tables,
                           int64_t max_blocks_per_seq,
                           const int32_t *context_lens, double scale,
                           const int64_t *pairs, int64_t num_pairs, double *out)
{
    if (dtype != 0 && dtype != 1)
        return -1;
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0 || block_size <= 0)
        return -1;
    int64_t total = pairs ? num_pairs : num_seqs * num_q_heads;
    int err = 0;

#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int64_t i = 0; i < total; ++i) {
        int64_t seq = pairs ? pairs[2 * i] : i / num_q_heads;
        int64_t head = pairs ? pairs[2 * i + 1] : i % num_q_heads;
        double *o = out + i * head_dim;
        if (seq < 0 || seq >= num_seqs || head < 0 || head >= num_q_heads) {
            err |= 1;
            continue;
        }
        int64_t ctx = context_lens[seq];
        double m, l;
        if (oracle_attention_range(dtype, q, num_q_heads, k_cache, v_cache,
                                   num_blocks, block_size, num_kv_heads,
                                   head_dim, block_tables, max_blocks_per_seq,
                                   scale, seq, head, 0, ctx, &m, &l, o)) {
            err |= 1;
            continue;
        }
        if (l > 0.0) {
            for (int64_t d = 0; d < head_dim; ++d)
                o[d] = o[d] / l;
        }
    }
    return err ? -1 : 0;
}

/*
 * Log-sum-exp merge of n partial results (m_j natural-log domain, l_j, o_j
 * unnormalised):  M = max m_j,  L = sum l_j e^{m_j - M},
 * out = sum o_j e^{m_j - M} / L.  Parts with m_j = -inf carry weight 0.
 */
int oracle_lse_merge(int64_t n, const double *m, const double *l,
                     const double *o, int64_t head_dim, double *out)
{
    double big = -INFINITY;
    for (int64_t j = 0; j < n; ++j)
        if (m[j] > big)
            big = m[j];
    for (int64_t d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    if (big == -INFINITY)
        return 0;
    double total = 0.0;
    for (int64_t j = 0; j < n; ++j) {
        double w = m[j] == -INFINITY ? 0.0 : exp(m[j] - big);
        total += l[j] * w;
        for (int64_t d = 0; d < head_dim; ++d)
            out[d] += o[j * head_dim + d] * w;
    }
    for (int64_t d = 0; d < head_dim; ++d)
        out[d] /= total;
    return 0;
}

int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n)
{
#ifdef _OPENMP
    if (n > 0)
        omp_set_num_threads(n);
#else
    (void)n;
#endif
}

/*
 * Mark every slot (block * bs + row) that holds a position p < lens[s] of some
 * sequence s: mask[slot] = 1.  Used by tests to poison every other slot.
 * Returns -1 if a needed table entry is outside [0, num_blocks).
 */
int oracle_mark_slots(const int32_t *block_tables, int64_t num_seqs,
                      int64_t max_blocks_per_seq, const int32_t *lens,
                      int64_t block_size, int64_t num_blocks, uint8_t *mask)
{
    for (int64_t s = 0; s < num_seqs; ++s) {
        const int32_t *row = block_tables + s * max_blocks_per_seq;
        for (int64_t p = 0; p < lens[s]; ++p) {
            int64_t b = row[p / block_size];
            if (b < 0 || b >= num_blocks)
                return -1;
            mask[b * block_size + p % block_size] = 1;
        }
    }
    return 0;
}

/*
 * Copy-on-write support: copy whole physical blocks (all KV heads, all rows)
 * src -> dst for each (src, dst) pair, in order.  A block is
 * kv_heads * block_size * head_dim 16-bit values, contiguous in the pool.
 * Sharing pages between requests with a common prefix is the pages' idea
 * (adilsher.pro post, "The Elegant Fix: Paged Attention"); a writer of a
 * shared page gets a private copy first (the plain reading of sharing with
 * appends).  Returns -1 if an id is outside [0, num_blocks).
 */
int oracle_copy_blocks(uint16_t *cache, int64_t num_blocks, int64_t block_elems,
                       const int32_t *pairs, int64_t num_pairs)
{
    for (int64_t i = 0; i < num_pairs; ++i) {
        int64_t src = pairs[2 * i], dst = pairs[2 * i + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks)
            return -1;
        memmove(cache + dst * block_elems, cache + src * block_elems,
                (size_t)block_elems * sizeof(uint16_t));
    }
    return 0;
}

/*
 * Chunked prefill attention ("LLM Inference: KV Cache, Batching &
 * Scheduling", cariara.com, section "Chunked prefill": a prompt is split
 * into fixed-size chunks interleaved with decode steps).  Sequence s has
 * n_s = query_start[s+1] - query_start[s] new query tokens whose K/V are
 * already in the cache at positions ctx_s - n_s .. ctx_s - 1; query i of the
 * chunk attends to positions 0 .. ctx_s - n_s + i (causal).  A decode
 * sequence is a chunk of one.  q and out are [T][Hq][D] with
 * T = query_start[B]; out is fp64.  Returns -1 on inconsistent lengths.
 */
int oracle_prefill_attention(int dtype, const uint16_t *q, int64_t num_tokens,
                             int64_t num_seqs, int64_t num_q_heads,
                             const uint16_t *k_cache, const uint16_t *v_cache,
                             int64_t num_blocks, int64_t block_size,
                             int64_t num_kv_heads, int64_t head_dim,
                             const int32_t *block_tables, int64_t max_blocks_per_seq,
                             const int32_t *query_start, const int32_t *context_lens,
                             double scale, double *out)
{
    if (query_start[0] != 0 || query_start[num_seqs] != num_tokens)
        return -1;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int64_t s = 0; s < num_seqs; ++s) {
        int64_t n = query_start[s + 1] - query_start[s];
        int64_t ctx = context_lens[s];
        if (n < 0 || ctx < n) {
            err |= 1;
            continue;
        }
        for (int64_t i = 0; i < n; ++i) {
            int64_t tok = query_start[s] + i;
            int64_t window = ctx - n + i + 1;     /* positions 0 .. ctx - n + i */
            for (int64_t h = 0; h < num_q_heads; ++h) {
                double m, l;
                double *o = out + (tok * num_q_heads + h) * head_dim;
                /* the query row of token tok, head h sits at q[tok][h]: call
                 * the range routine with the token's row as "sequence" */
                if (oracle_attention_range(dtype, q + tok * num_q_heads * head_dim, num_q_heads,
                                           k_cache, v_cache, num_blocks, block_size,
                                           num_kv_heads, head_dim,
                                           block_tables + s * max_blocks_per_seq,
                                           max_blocks_per_seq, scale, 0, h, 0, window,
                                           &m, &l, o)) {
                    err |= 1;
                    continue;
                }
                if (l > 0.0)
                    for (int64_t d = 0; d < head_dim; ++d)
                        o[d] /= l;
            }
        }
    }
    return err ? -1 : 0;
}

/* ---- FP8 E4M3 KV cache -----------------------------------------------------
 * The pages leave quantization open ("How do quantization and batching
 * strategy interact?", adilsher.pro post, "What I'm Still Figuring Out").
 * Format (OCP FP8 E4M3, no infinities): bits s eeee mmm; e = 0: value
 * m * 2^-9; e >= 1: (1 + m/8) * 2^(e-7); e = 15, m = 7 is NaN; largest
 * finite 448.  Each appended (token, KV head) row gets one fp32 scale:
 * scale = amax / 448 (1 if amax == 0), code_d = nearest code to x_d / scale
 * (ties to the even code, magnitudes past 448 saturate), both divisions in
 * fp32 with round-to-nearest.  A cached value is value(code) * scale.
 * Pools: codes [NB][Hkv][bs][D] (bytes), scales [NB][Hkv][bs] (fp32).
 */
double oracle_e4m3_value(uint8_t code)
{
    int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v;
    if (e == 15 && m == 7)
        return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);
    else
        v = ldexp(1.0 + m / 8.0, e - 7);
    return sign ? -v : v;
}

uint8_t oracle_e4m3_quantize(float y)
{
    /* nearest finite code by exhaustive search over the 127 magnitudes */
    double a = fabs((double)y);
    int best = 0;
    double best_err = INFINITY;
    for (int c = 0; c <= 0x7e; ++c) {
        double err = fabs(oracle_e4m3_value((uint8_t)c) - a);
        if (err < best_err || (err == best_err && (c & 1) == 0 && (best & 1) == 1)) {
            best = c;
            best_err = err;
        }
    }
    if (a >= 448.0)
        best = 0x7e;
    return (uint8_t)(best | (y < 0 ? 0x80 : 0));
}

float oracle_e4m3_row_scale(const uint16_t *row, int64_t head_dim, int dtype)
{
    float amax = 0.0f;
    for (int64_t d = 0; d < head_dim; ++d) {
        float x = (float)decode16(dtype, row[d]);
        if (fabsf(x) > amax)
            amax = fabsf(x);
    }
    return amax > 0.0f ? amax / 448.0f : 1.0f;
}

int oracle_append_e4m3(uint8_t *cache, float *scales, int64_t num_blocks, int64_t kv_heads,
                       int64_t block_size, int64_t head_dim, const uint16_t *new_kv,
                       int new_dtype, const int64_t *slot_mapping, int64_t num_tokens)
{
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        int64_t block = slot / block_size;
        int64_t row = slot % block_size;
        if (block >= num_blocks)
            return -1;
        for (int64_t h = 0; h < kv_heads; ++h) {
            const uint16_t *xrow = new_kv + (t * kv_heads + h) * head_dim;
            int64_t r = (block * kv_heads + h) * block_size + row;
            float sc = oracle_e4m3_row_scale(xrow, head_dim, new_dtype);
            scales[r] = sc;
            for (int64_t d = 0; d < head_dim; ++d) {
                float y = (float)decode16(new_dtype, xrow[d]) / sc;
                cache[r * head_dim + d] = oracle_e4m3_quantize(y);
            }
        }
    }
    return 0;
}

static int gather_row_e4m3(const uint8_t *cache, const float *scales, int64_t num_blocks,
                           int64_t kv_heads, int64_t block_size, int64_t head_dim,
                           const int32_t *table_row, int64_t pos, int64_t g, double *dst)
{
    int64_t phys = table_row[pos / block_size];
    int64_t row = pos % block_size;
    if (phys < 0 || phys >= num_blocks)
        return -1;
    int64_t r = (phys * kv_heads + g) * block_size + row;
    for (int64_t d = 0; d < head_dim; ++d)
        dst[d] = oracle_e4m3_value(cache[r * head_dim + d]) * (double)scales[r];
    return 0;
}

/* Decode attention over E4M3 pools: the definition of
 * oracle_paged_attention with every K/V row dequantized (value * scale). */
int oracle_paged_attention_e4m3(int q_dtype, const uint16_t *q, int64_t num_seqs,
                                int64_t num_q_heads, const uint8_t *k_cache, const float *k_scales,
                                const uint8_t *v_cache, const float *v_scales,
                                int64_t num_blocks, int64_t block_size, int64_t num_kv_heads,
                                int64_t head_dim, const int32_t *block_tables,
                                int64_t max_blocks_per_seq, const int32_t *context_lens,
                                double scale, double *out)
{
    if (num_kv_heads <= 0 || num_q_heads % num_kv_heads != 0)
        return -1;
    int64_t group = num_q_heads / num_kv_heads;
    int err = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int64_t i = 0; i < num_seqs * num_q_heads; ++i) {
        int64_t seq = i / num_q_heads, head = i % num_q_heads, g = head / group;
        int64_t ctx = context_lens[seq];
        double *o = out + i * head_dim;
        const int32_t *table_row = block_tables + seq * max_blocks_per_seq;
        for (int64_t d = 0; d < head_dim; ++d)
            o[d] = 0.0;
        if (ctx <= 0)
            continue;
        double *qd = malloc(sizeof(double) * head_dim);
        double *row = malloc(sizeof(double) * head_dim);
        double *z = malloc(sizeof(double) * ctx);
        if (!qd || !row || !z) {
            err |= 1;
            free(qd);
            free(row);
            free(z);
            continue;
        }
        for (int64_t d = 0; d < head_dim; ++d)
            qd[d] = decode16(q_dtype, q[(seq * num_q_heads + head) * head_dim + d]);
        double m = -INFINITY;
        for (int64_t p = 0; p < ctx && !err; ++p) {
            if (gather_row_e4m3(k_cache, k_scales, num_blocks, num_kv_heads, block_size, head_dim,
                                table_row, p, g, row)) {
                err |= 1;
                break;
            }
            double dot = 0.0;
            for (int64_t d = 0; d < head_dim; ++d)
                dot += qd[d] * row[d];
            z[p] = scale * dot;
            if (z[p] > m)
                m = z[p];
        }
        double l = 0.0;
        for (int64_t p = 0; p < ctx && !err; ++p) {
            double w = exp(z[p] - m);
            l += w;
            if (gather_row_e4m3(v_cache, v_scales, num_blocks, num_kv_heads, block_size, head_dim,
                                table_row, p, g, row)) {
                err |= 1;
                break;
            }
            for (int64_t d = 0; d < head_dim; ++d)
                o[d] += w * row[d];
        }
        if (l > 0.0)
            for (int64_t d = 0; d < head_dim; ++d)
                o[d] /= l;
        free(qd);
        free(row);
        free(z);
    }
    return err ? -1 : 0;
}

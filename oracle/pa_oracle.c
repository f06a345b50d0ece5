/*
 * CPU oracle for the paged-KV attention step.  TEST INFRASTRUCTURE ONLY:
 * only tests/, __graft_entry__.smoke() and bench.py's cpu_baseline /
 * reference leg may load this library.  It shares no code, header, table or
 * helper with the CUDA path; it is a plain, slow, obviously correct statement
 * of what the path computes, in fp64.
 *
 * What it follows (pages are cited by title and section):
 *  - "vLLM 学习笔记 01：一个请求在 vLLM 里的一生" §1.5 (分页式 KV 缓存): the KV
 *    cache is cut into fixed blocks of 16 tokens, and each request owns a
 *    block table listing which physical block holds its 1st, 2nd, 3rd ...
 *    block; blocks need not be contiguous.
 *  - same page, §1.6 (前向计算：不补齐的批): all tokens of a step are
 *    concatenated into one unpadded stream; the attention op is told where
 *    each segment starts and ends (segments cannot see one another), and, per
 *    token, the slot (block and position) its K/V goes to.
 *  - same page, §1.4 and §2.1: a request tracks computed vs total tokens, so
 *    a segment's seq_len counts the tokens scheduled this step, and a
 *    prefill chunk reads the context cached by earlier chunks.
 *  - same page, §2.5 (prefill/decode disaggregation): a prefill instance
 *    produces a request's full KV cache and a connector moves it to a decode
 *    instance; kv_export / kv_import state the local half, a request's K/V
 *    between its blocks and one contiguous buffer.
 *  - "Inside vLLM: Anatomy of a High-Throughput LLM Inference System"
 *    (Chinese translation), section "LLM 引擎构造函数" (engine constructor),
 *    KV cache manager paragraph: one block of a standard (non-MLA) layer holds
 *    K and V of block_size (default 16) tokens for every kv head, i.e.
 *    2 * block_size * kv_heads * head_size * dtype bytes.
 *
 * Readings where the pages are silent (each is stated where it is used):
 *  - cache layout [num_blocks][block_size][kv_heads][head_dim], K and V in two
 *    separate buffers; slot = block_id * block_size + offset;
 *  - a negative slot means "skip this token";
 *  - causal alignment is bottom-right: query j of a segment with q_len L and
 *    seq_len n sits at position n - L + j and sees keys 0 .. n - L + j;
 *  - query head h reads kv head h / (num_q_heads / num_kv_heads) (GQA);
 *  - bf16 values are widened exactly to fp64 and all arithmetic is fp64.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum {
    ORACLE_OK = 0,
    ORACLE_ERR_ARG = 1,     /* bad sizes or null pointers */
    ORACLE_ERR_SLOT = 2,    /* slot outside the pool */
    ORACLE_ERR_SEGMENT = 3, /* cu_seqlens not monotone, or q_len > seq_len */
    ORACLE_ERR_BLOCK = 4,   /* a block id the segment needs is outside the pool */
    ORACLE_ERR_ROW = 5,     /* a requested output row does not exist */
    ORACLE_ERR_NOMEM = 6
};

/* bf16 is the top half of an IEEE binary32; widening is exact. */
static double bf16_to_f64(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * reshape_and_cache: for every token t whose slot s = slot_mapping[t] is not
 * negative, copy k[t] (all kv heads, all dims) into k_cache at block
 * s / block_size, row s % block_size, and v[t] into v_cache likewise.  The
 * copy is bitwise.  Every other cache entry is left as it was.
 */
int oracle_reshape_and_cache(const uint16_t *k, const uint16_t *v,
                             const int64_t *slot_mapping, int64_t num_tokens,
                             int num_kv_heads, int head_dim,
                             uint16_t *k_cache, uint16_t *v_cache,
                             int64_t num_blocks, int block_size)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        num_blocks <= 0 || block_size <= 0)
        return ORACLE_ERR_ARG;
    if (num_tokens > 0 && (!k || !v || !slot_mapping || !k_cache || !v_cache))
        return ORACLE_ERR_ARG;
    const int64_t token_elems = (int64_t)num_kv_heads * head_dim;
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t s = slot_mapping[t];
        if (s < 0)
            continue;
        if (s >= num_blocks * block_size)
            return ORACLE_ERR_SLOT;
    }
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t s = slot_mapping[t];
        if (s < 0)
            continue;
        int64_t block = s / block_size;
        int64_t offset = s % block_size;
        int64_t dst = (block * block_size + offset) * token_elems;
        for (int64_t e = 0; e < token_elems; ++e) {
            k_cache[dst + e] = k[t * token_elems + e];
            v_cache[dst + e] = v[t * token_elems + e];
        }
    }
    return ORACLE_OK;
}

/*
 * kv_export / kv_import: request i (0 <= i < num_seqs) owns buffer rows
 * cu_tokens[i] .. cu_tokens[i + 1] - 1; its token p is row p of that range
 * and row p % block_size of cache block block_tables[i][p / block_size].
 * Export copies every such token's K and V (all kv heads) from the caches to
 * the buffers, import the other way; bitwise.  Nothing else is touched.
 */
static int kv_transfer(int do_export, uint16_t *k_cache, uint16_t *v_cache, int64_t num_blocks,
                       int block_size, int num_kv_heads, int head_dim, const int32_t *block_tables,
                       int max_blocks_per_seq, const int32_t *cu_tokens, int num_seqs,
                       uint16_t *k_buf, uint16_t *v_buf)
{
    if (num_seqs < 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 || block_size <= 0 ||
        max_blocks_per_seq < 0)
        return ORACLE_ERR_ARG;
    if (num_seqs == 0)
        return ORACLE_OK;
    if (!k_cache || !v_cache || !block_tables || !cu_tokens || !k_buf || !v_buf)
        return ORACLE_ERR_ARG;
    if (cu_tokens[0] != 0)
        return ORACLE_ERR_SEGMENT;
    for (int i = 0; i < num_seqs; ++i) {
        int n = cu_tokens[i + 1] - cu_tokens[i];
        if (n < 0 || (int64_t)n > (int64_t)max_blocks_per_seq * block_size)
            return ORACLE_ERR_SEGMENT;
        for (int b = 0; b * block_size < n; ++b) {
            int32_t id = block_tables[(int64_t)i * max_blocks_per_seq + b];
            if (id < 0 || id >= num_blocks)
                return ORACLE_ERR_BLOCK;
        }
    }
    const int64_t token_elems = (int64_t)num_kv_heads * head_dim;
    for (int i = 0; i < num_seqs; ++i) {
        for (int p = 0; p < cu_tokens[i + 1] - cu_tokens[i]; ++p) {
            int64_t block = block_tables[(int64_t)i * max_blocks_per_seq + p / block_size];
            int64_t cache_row = block * block_size + p % block_size;
            int64_t buf_row = (int64_t)cu_tokens[i] + p;
            for (int64_t e = 0; e < token_elems; ++e) {
                if (do_export) {
                    k_buf[buf_row * token_elems + e] = k_cache[cache_row * token_elems + e];
                    v_buf[buf_row * token_elems + e] = v_cache[cache_row * token_elems + e];
                } else {
                    k_cache[cache_row * token_elems + e] = k_buf[buf_row * token_elems + e];
                    v_cache[cache_row * token_elems + e] = v_buf[buf_row * token_elems + e];
                }
            }
        }
    }
    return ORACLE_OK;
}

int oracle_kv_export(const uint16_t *k_cache, const uint16_t *v_cache, int64_t num_blocks, int block_size,
                     int num_kv_heads, int head_dim, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *cu_tokens, int num_seqs, uint16_t *k_out, uint16_t *v_out)
{
    return kv_transfer(1, (uint16_t *)k_cache, (uint16_t *)v_cache, num_blocks, block_size, num_kv_heads,
                       head_dim, block_tables, max_blocks_per_seq, cu_tokens, num_seqs, k_out, v_out);
}

int oracle_kv_import(const uint16_t *k_in, const uint16_t *v_in, int64_t num_blocks, int block_size,
                     int num_kv_heads, int head_dim, const int32_t *block_tables, int max_blocks_per_seq,
                     const int32_t *cu_tokens, int num_seqs, uint16_t *k_cache, uint16_t *v_cache)
{
    return kv_transfer(0, k_cache, v_cache, num_blocks, block_size, num_kv_heads, head_dim, block_tables,
                       max_blocks_per_seq, cu_tokens, num_seqs, (uint16_t *)k_in, (uint16_t *)v_in);
}

typedef struct {
    const uint16_t *q, *k_cache, *v_cache;
    const int32_t *block_tables, *cu_seqlens_q, *seq_lens;
    int num_seqs, num_q_heads, num_kv_heads, head_dim;
    int64_t num_blocks;
    int max_blocks_per_seq, block_size;
    double scale;
} problem;

/* The head_dim-long K (or V) vector of kv head g at logical position pos of
 * segment i, found through the segment's block table: logical block
 * pos / block_size is physical block block_tables[i][pos / block_size], and
 * the token sits at row pos % block_size of that block. */
static const uint16_t *cached_row(const problem *P, const uint16_t *cache, int i,
                                  int64_t pos, int g)
{
    int32_t block = P->block_tables[(int64_t)i * P->max_blocks_per_seq +
                                    pos / P->block_size];
    int64_t offset = pos % P->block_size;
    return cache + (((int64_t)block * P->block_size + offset) * P->num_kv_heads + g) *
                       P->head_dim;
}

/*
 * One output row: query j (0 <= j < q_len) of segment i, query head h.
 * Its absolute position is p = seq_len - q_len + j; it attends to keys
 * 0 .. p of its own segment only.  scores z_tau = scale * <q, K[tau]>;
 * out = sum_tau softmax(z)_tau * V[tau], with the softmax taken as
 * exp(z - max z) / sum exp(z - max z).
 */
static void attend_row(const problem *P, int i, int j, int h, double *scores,
                       double *out)
{
    const int64_t n = P->seq_lens[i];
    const int64_t L = (int64_t)P->cu_seqlens_q[i + 1] - P->cu_seqlens_q[i];
    const int64_t t = (int64_t)P->cu_seqlens_q[i] + j;
    const int64_t p = n - L + j;
    const int group = P->num_q_heads / P->num_kv_heads;
    const int g = h / group;
    const uint16_t *qrow = P->q + (t * P->num_q_heads + h) * P->head_dim;
    const int D = P->head_dim;

    double zmax = -INFINITY;
    for (int64_t tau = 0; tau <= p; ++tau) {
        const uint16_t *krow = cached_row(P, P->k_cache, i, tau, g);
        double dot = 0.0;
        for (int d = 0; d < D; ++d)
            dot += bf16_to_f64(qrow[d]) * bf16_to_f64(krow[d]);
        scores[tau] = P->scale * dot;
        if (scores[tau] > zmax)
            zmax = scores[tau];
    }
    double denom = 0.0;
    for (int64_t tau = 0; tau <= p; ++tau) {
        scores[tau] = exp(scores[tau] - zmax);
        denom += scores[tau];
    }
    for (int d = 0; d < D; ++d)
        out[d] = 0.0;
    for (int64_t tau = 0; tau <= p; ++tau) {
        const uint16_t *vrow = cached_row(P, P->v_cache, i, tau, g);
        double w = scores[tau] / denom;
        for (int d = 0; d < D; ++d)
            out[d] += w * bf16_to_f64(vrow[d]);
    }
}

/* Segment that holds flat token t (cu_seqlens_q is non-decreasing). */
static int segment_of(const problem *P, int64_t t)
{
    for (int i = 0; i < P->num_seqs; ++i)
        if (t >= P->cu_seqlens_q[i] && t < P->cu_seqlens_q[i + 1])
            return i;
    return -1;
}

/*
 * Varlen paged attention.  If rows is NULL, every output row is computed and
 * out is [num_tokens][num_q_heads][head_dim].  Otherwise rows holds n_rows
 * flat row ids (token * num_q_heads + head) and out is [n_rows][head_dim].
 * threads <= 0 uses the OpenMP default.
 */
int oracle_attention_varlen(const uint16_t *q, const uint16_t *k_cache,
                            const uint16_t *v_cache, const int32_t *block_tables,
                            const int32_t *cu_seqlens_q, const int32_t *seq_lens,
                            int num_seqs, int num_q_heads, int num_kv_heads,
                            int head_dim, int64_t num_blocks,
                            int max_blocks_per_seq, int block_size, double scale,
                            const int64_t *rows, int64_t n_rows, double *out,
                            int threads)
{
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        num_blocks <= 0 || max_blocks_per_seq < 0 || block_size <= 0 ||
        num_q_heads % num_kv_heads != 0 || !cu_seqlens_q || !seq_lens || !out)
        return ORACLE_ERR_ARG;
    problem P = {q, k_cache, v_cache, block_tables, cu_seqlens_q, seq_lens,
                 num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks,
                 max_blocks_per_seq, block_size, scale};

    /* Check what the rows read: segment bounds and every block id in use. */
    if (cu_seqlens_q[0] != 0)
        return ORACLE_ERR_SEGMENT;
    int64_t max_n = 0;
    for (int i = 0; i < num_seqs; ++i) {
        int64_t L = (int64_t)cu_seqlens_q[i + 1] - cu_seqlens_q[i];
        int64_t n = seq_lens[i];
        if (L < 0 || n < L)
            return ORACLE_ERR_SEGMENT;
        if (L == 0)
            continue;
        int64_t used = (n + block_size - 1) / block_size;
        if (used > max_blocks_per_seq)
            return ORACLE_ERR_BLOCK;
        for (int64_t b = 0; b < used; ++b) {
            int32_t id = block_tables[(int64_t)i * max_blocks_per_seq + b];
            if (id < 0 || id >= num_blocks)
                return ORACLE_ERR_BLOCK;
        }
        if (n > max_n)
            max_n = n;
    }
    const int64_t num_tokens = cu_seqlens_q[num_seqs];
    const int64_t total = rows ? n_rows : num_tokens * num_q_heads;
    if (total > 0 && (!q || !k_cache || !v_cache || !block_tables))
        return ORACLE_ERR_ARG;
    if (rows)
        for (int64_t r = 0; r < n_rows; ++r)
            if (rows[r] < 0 || rows[r] >= num_tokens * num_q_heads)
                return ORACLE_ERR_ROW;

#ifdef _OPENMP
    if (threads <= 0)
        threads = omp_get_max_threads();
#else
    threads = 1;
#endif
    int failed = 0;
#pragma omp parallel num_threads(threads)
    {
        double *scores = (double *)malloc(sizeof(double) * (size_t)(max_n > 0 ? max_n : 1));
        if (!scores) {
#pragma omp atomic write
            failed = 1;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t r = 0; r < total; ++r) {
            if (!scores)
                continue;
            int64_t flat = rows ? rows[r] : r;
            int64_t t = flat / num_q_heads;
            int h = (int)(flat % num_q_heads);
            int i = segment_of(&P, t);
            int j = (int)(t - cu_seqlens_q[i]);
            attend_row(&P, i, j, h, scores, out + r * head_dim);
        }
        free(scores);
    }
    return failed ? ORACLE_ERR_NOMEM : ORACLE_OK;
}

/* Threads an OpenMP parallel region would use by default. */
int oracle_default_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * oracle.c -- the fp64 CPU oracle for paged decode attention.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product library calls, links or
 * includes this file; only the tests, the package's smoke check and the
 * benchmark's CPU-baseline leg use it. It shares no code, header or
 * constant with the CUDA path.
 *
 * What it computes, and where the pages define it:
 *
 *  - Attention itself is unchanged by paging: the output is
 *    softmax(q K^T / sqrt(d)) V over the sequence's whole history
 *    (page "大语言模型推理内存管理算法 paged attention", section 5 formula
 *    and section 6 "the attention formula is not changed"; page "08.
 *    PagedAttention：把 KV Cache 分页管理", section "它没有解决什么": every
 *    decode step still reads all history).
 *  - A token's K/V is found by taking its logical block (position /
 *    block_size) through the sequence's block table to a physical block
 *    (first page, sections 2, 5 and 8; third page, section
 *    "借用操作系统的办法：分页").
 *  - A token's slot is block_table[logical block] * block_size + offset in
 *    the block, and the write kernel stores each new token's K and V at its
 *    slot (third page, section "为什么叫 PagedAttention").
 *  - Copy-on-write copies a shared block's contents into a newly allocated
 *    block (page "PagedAttention 核心思想解析", section 2.3).
 *  - Partial results computed per part of the KV sequence are merged
 *    (second page, section 2.2). The merge here is the log-sum-exp
 *    combination of per-partition (max, sum, weighted V) states, which is
 *    algebraically identical to the unpartitioned softmax.
 *
 * Memory layout read through accessors (the pages give none; this is the
 * reading the whole build uses): K and V pools are separate arrays of shape
 * [num_blocks][num_kv_heads][block_size][head_dim]; q and out are
 * [num_seqs][num_q_heads][head_dim]; block tables are int32
 * [num_seqs][max_blocks_per_seq]; query head h reads KV head
 * h / (num_q_heads / num_kv_heads) (grouped-query attention, first page,
 * section 6 table).
 *
 * Precision: every stored 16-bit value is widened exactly to double, all
 * arithmetic is double, results are left unrounded.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_F16 0
#define ORC_BF16 1

#define ORC_OK 0
#define ORC_BAD_ARG -1
#define ORC_BAD_BLOCK -2
#define ORC_BAD_SLOT -3

/* IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits. */
double oracle_f16_to_double(uint16_t h)
{
    int sign = (h >> 15) & 1;
    int e = (h >> 10) & 0x1f;
    int f = h & 0x3ff;
    double mag;
    if (e == 0)
        mag = ldexp((double)f, -24);                 /* subnormal: f * 2^-24 */
    else if (e == 31)
        mag = f ? NAN : INFINITY;
    else
        mag = ldexp((double)(1024 + f), e - 25);     /* (1 + f/2^10) * 2^(e-15) */
    return sign ? -mag : mag;
}

/* bfloat16: the upper 16 bits of IEEE binary32 -- 1 sign, 8 exponent bits
 * (bias 127), 7 fraction bits. */
double oracle_bf16_to_double(uint16_t b)
{
    int sign = (b >> 15) & 1;
    int e = (b >> 7) & 0xff;
    int f = b & 0x7f;
    double mag;
    if (e == 0)
        mag = ldexp((double)f, -133);                /* subnormal: f * 2^(-126-7) */
    else if (e == 255)
        mag = f ? NAN : INFINITY;
    else
        mag = ldexp((double)(128 + f), e - 134);     /* (1 + f/2^7) * 2^(e-127) */
    return sign ? -mag : mag;
}

static double widen(uint16_t bits, int dtype)
{
    return dtype == ORC_BF16 ? oracle_bf16_to_double(bits) : oracle_f16_to_double(bits);
}

/* Slot of logical position `pos` of a sequence whose block table row is
 * `table_row`: the physical block that holds the position, times the block
 * size, plus the position's offset inside its block. */
int64_t oracle_slot(const int32_t *table_row, int64_t pos, int block_size)
{
    int64_t logical_block = pos / block_size;
    int64_t offset = pos % block_size;
    return (int64_t)table_row[logical_block] * block_size + offset;
}

/* Index of element (block, kv_head, offset, d) in a K or V pool. */
static size_t pool_index(int64_t block, int kv_head, int offset, int d,
                         int num_kv_heads, int block_size, int head_dim)
{
    return (((size_t)block * num_kv_heads + kv_head) * block_size + offset) * head_dim + d;
}

/* Store the K and V rows of `num_tokens` new tokens at their slots.
 * k_new, v_new: [num_tokens][num_kv_heads][head_dim] 16-bit patterns.
 * A negative slot marks a padding token, which is skipped. */
int oracle_reshape_and_cache(const uint16_t *k_new, const uint16_t *v_new,
                             const int64_t *slot_mapping, int num_tokens,
                             uint16_t *k_cache, uint16_t *v_cache,
                             int num_blocks, int num_kv_heads, int block_size, int head_dim)
{
    if (num_tokens < 0 || num_kv_heads <= 0 || block_size <= 0 || head_dim <= 0)
        return ORC_BAD_ARG;
    for (int t = 0; t < num_tokens; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        if (slot >= (int64_t)num_blocks * block_size)
            return ORC_BAD_SLOT;
        int64_t block = slot / block_size;
        int offset = (int)(slot % block_size);
        for (int h = 0; h < num_kv_heads; ++h) {
            for (int d = 0; d < head_dim; ++d) {
                size_t src = ((size_t)t * num_kv_heads + h) * head_dim + d;
                size_t dst = pool_index(block, h, offset, d, num_kv_heads, block_size, head_dim);
                k_cache[dst] = k_new[src];
                v_cache[dst] = v_new[src];
            }
        }
    }
    return ORC_OK;
}

/* Copy whole blocks (every KV head, every slot, K and V) for each
 * (src, dst) pair of `block_pairs` ([num_pairs][2]), in pair order. */
int oracle_copy_blocks(uint16_t *k_cache, uint16_t *v_cache, const int64_t *block_pairs,
                       int num_pairs, int num_blocks, int num_kv_heads, int block_size,
                       int head_dim)
{
    size_t block_elems = (size_t)num_kv_heads * block_size * head_dim;
    for (int p = 0; p < num_pairs; ++p) {
        int64_t src = block_pairs[2 * p], dst = block_pairs[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks)
            return ORC_BAD_BLOCK;
        for (size_t i = 0; i < block_elems; ++i) {
            k_cache[(size_t)dst * block_elems + i] = k_cache[(size_t)src * block_elems + i];
            v_cache[(size_t)dst * block_elems + i] = v_cache[(size_t)src * block_elems + i];
        }
    }
    return ORC_OK;
}

/* Gather the logical rows [0, n) of one (sequence, KV head) from a pool into
 * a contiguous double array [n][head_dim]. Returns ORC_BAD_BLOCK if the
 * table names a block outside the pool. */
static int gather_rows(double *dst, const uint16_t *pool, const int32_t *table_row, int n,
                       int kv_head, int num_blocks, int num_kv_heads, int block_size,
                       int head_dim, int dtype)
{
    for (int t = 0; t < n; ++t) {
        int64_t slot = oracle_slot(table_row, t, block_size);
        int64_t block = slot / block_size;
        int offset = (int)(slot % block_size);
        if (block < 0 || block >= num_blocks)
            return ORC_BAD_BLOCK;
        for (int d = 0; d < head_dim; ++d)
            dst[(size_t)t * head_dim + d] =
                widen(pool[pool_index(block, kv_head, offset, d, num_kv_heads, block_size,
                                      head_dim)], dtype);
    }
    return ORC_OK;
}

/* Textbook attention of one query row over n contiguous K/V rows:
 * s_t = scale * q.k_t, w_t = exp(s_t - max s), out = sum w_t v_t / sum w_t.
 * Subtracting the max changes no value of the softmax; it keeps exp finite.
 * n == 0 yields zeros. */
static void attend_rows(double *out, const double *q, const double *K, const double *V, int n,
                        int head_dim, double scale, double *s)
{
    for (int d = 0; d < head_dim; ++d)
        out[d] = 0.0;
    if (n == 0)
        return;
    double m = -INFINITY;
    for (int t = 0; t < n; ++t) {
        double dot = 0.0;
        for (int d = 0; d < head_dim; ++d)
            dot += q[d] * K[(size_t)t * head_dim + d];
        s[t] = scale * dot;
        if (s[t] > m)
            m = s[t];
    }
    double denom = 0.0;
    for (int t = 0; t < n; ++t) {
        double w = exp(s[t] - m);
        denom += w;
        for (int d = 0; d < head_dim; ++d)
            out[d] += w * V[(size_t)t * head_dim + d];
    }
    for (int d = 0; d < head_dim; ++d)
        out[d] /= denom;
}

static int check_shapes(int num_seqs, int num_q_heads, int num_kv_heads, int head_dim,
                        int block_size, int num_blocks, int max_blocks_per_seq)
{
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        block_size <= 0 || num_blocks <= 0 || max_blocks_per_seq <= 0)
        return ORC_BAD_ARG;
    if (num_q_heads % num_kv_heads)
        return ORC_BAD_ARG;
    return ORC_OK;
}

static int set_threads(int num_threads)
{
#ifdef _OPENMP
    if (num_threads > 0)
        return num_threads;
    return omp_get_max_threads();
#else
    (void)num_threads;
    return 1;
#endif
}

/* Paged decode attention for a batch, one query token per sequence.
 * out: double [num_seqs][num_q_heads][head_dim].
 * For every (sequence b, query head h): gather the n = context_lens[b]
 * rows of KV head h / group through the block table, then attend.
 * num_threads: OpenMP threads over (sequence, q head); 0 = all available. */
int oracle_decode(double *out, const uint16_t *q, const uint16_t *k_cache,
                  const uint16_t *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                  const int32_t *context_lens, int num_seqs, int num_q_heads, int num_kv_heads,
                  int head_dim, int block_size, int num_blocks, float scale, int dtype,
                  int num_threads)
{
    int rc = check_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                          num_blocks, max_blocks_per_seq);
    if (rc)
        return rc;
    for (int b = 0; b < num_seqs; ++b)
        if (context_lens[b] < 0 || context_lens[b] > max_blocks_per_seq * block_size)
            return ORC_BAD_ARG;
    int group = num_q_heads / num_kv_heads;
    int nthreads = set_threads(num_threads);
    int status = ORC_OK;
    long long units = (long long)num_seqs * num_q_heads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (long long u = 0; u < units; ++u) {
        int b = (int)(u / num_q_heads), h = (int)(u % num_q_heads);
        int n = context_lens[b];
        int g = h / group;
        double *K = malloc(sizeof(double) * ((size_t)n * head_dim + 1));
        double *V = malloc(sizeof(double) * ((size_t)n * head_dim + 1));
        double *s = malloc(sizeof(double) * ((size_t)n + 1));
        double *qd = malloc(sizeof(double) * (size_t)head_dim);
        const int32_t *row = block_tables + (size_t)b * max_blocks_per_seq;
        int r1 = gather_rows(K, k_cache, row, n, g, num_blocks, num_kv_heads, block_size,
                             head_dim, dtype);
        int r2 = gather_rows(V, v_cache, row, n, g, num_blocks, num_kv_heads, block_size,
                             head_dim, dtype);
        if (r1 || r2) {
#ifdef _OPENMP
#pragma omp critical
#endif
            status = ORC_BAD_BLOCK;
        } else {
            for (int d = 0; d < head_dim; ++d)
                qd[d] = widen(q[((size_t)b * num_q_heads + h) * head_dim + d], dtype);
            attend_rows(out + ((size_t)b * num_q_heads + h) * head_dim, qd, K, V, n, head_dim,
                        (double)scale, s);
        }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
    (void)nthreads;
    return status;
}

/* Decode of a single (sequence, q head): the same definition as
 * oracle_decode, for checking sampled outputs of large batches. */
int oracle_decode_one(double *out, const uint16_t *q_row, const uint16_t *k_cache,
                      const uint16_t *v_cache, const int32_t *table_row, int context_len,
                      int kv_head, int num_kv_heads, int head_dim, int block_size,
                      int num_blocks, float scale, int dtype)
{
    int n = context_len;
    if (n < 0)
        return ORC_BAD_ARG;
    double *K = malloc(sizeof(double) * ((size_t)n * head_dim + 1));
    double *V = malloc(sizeof(double) * ((size_t)n * head_dim + 1));
    double *s = malloc(sizeof(double) * ((size_t)n + 1));
    double *qd = malloc(sizeof(double) * (size_t)head_dim);
    int rc = gather_rows(K, k_cache, table_row, n, kv_head, num_blocks, num_kv_heads,
                         block_size, head_dim, dtype);
    if (!rc)
        rc = gather_rows(V, v_cache, table_row, n, kv_head, num_blocks, num_kv_heads,
                         block_size, head_dim, dtype);
    if (!rc) {
        for (int d = 0; d < head_dim; ++d)
            qd[d] = widen(q_row[d], dtype);
        attend_rows(out, qd, K, V, n, head_dim, (double)scale, s);
    }
    free(K);
    free(V);
    free(s);
    free(qd);
    return rc;
}

/* Split-context decode: the KV sequence of every (sequence, q head) is cut
 * into partitions of `partition_tokens` consecutive positions. Partition p
 * yields its own max m_p, sum l_p = sum exp(s_t - m_p) and weighted sum
 * a_p = sum exp(s_t - m_p) v_t; the partial results are then merged:
 * M = max_p m_p, L = sum_p exp(m_p - M) l_p, out = sum_p exp(m_p - M) a_p / L.
 * If part_m / part_l / part_acc are non-NULL the per-partition states are
 * written there: part_m, part_l [num_seqs][num_q_heads][max_parts],
 * part_acc [num_seqs][num_q_heads][max_parts][head_dim], partitions past a
 * sequence's end left as m = -inf, l = 0, a = 0. */
int oracle_decode_partitioned(double *out, const uint16_t *q, const uint16_t *k_cache,
                              const uint16_t *v_cache, const int32_t *block_tables,
                              int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                              int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                              int num_blocks, float scale, int dtype, int partition_tokens,
                              int max_parts, double *part_m, double *part_l, double *part_acc,
                              int num_threads)
{
    int rc = check_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                          num_blocks, max_blocks_per_seq);
    if (rc)
        return rc;
    if (partition_tokens <= 0 || max_parts <= 0)
        return ORC_BAD_ARG;
    for (int b = 0; b < num_seqs; ++b) {
        if (context_lens[b] < 0 || context_lens[b] > max_blocks_per_seq * block_size)
            return ORC_BAD_ARG;
        if ((context_lens[b] + partition_tokens - 1) / partition_tokens > max_parts)
            return ORC_BAD_ARG;
    }
    int group = num_q_heads / num_kv_heads;
    int nthreads = set_threads(num_threads);
    int status = ORC_OK;
    long long units = (long long)num_seqs * num_q_heads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (long long u = 0; u < units; ++u) {
        int b = (int)(u / num_q_heads), h = (int)(u % num_q_heads);
        int n = context_lens[b];
        int g = h / group;
        const int32_t *row = block_tables + (size_t)b * max_blocks_per_seq;
        double *K = malloc(sizeof(double) * ((size_t)n * head_dim + 1));
        double *V = malloc(sizeof(double) * ((size_t)n * head_dim + 1));
        double *qd = malloc(sizeof(double) * (size_t)head_dim);
        double *m = malloc(sizeof(double) * (size_t)max_parts);
        double *l = malloc(sizeof(double) * (size_t)max_parts);
        double *a = calloc((size_t)max_parts * head_dim, sizeof(double));
        int r1 = gather_rows(K, k_cache, row, n, g, num_blocks, num_kv_heads, block_size,
                             head_dim, dtype);
        int r2 = gather_rows(V, v_cache, row, n, g, num_blocks, num_kv_heads, block_size,
                             head_dim, dtype);
        if (r1 || r2) {
#ifdef _OPENMP
#pragma omp critical
#endif
            status = ORC_BAD_BLOCK;
        } else {
            for (int d = 0; d < head_dim; ++d)
                qd[d] = widen(q[((size_t)b * num_q_heads + h) * head_dim + d], dtype);
            int parts = (n + partition_tokens - 1) / partition_tokens;
            for (int p = 0; p < max_parts; ++p) {
                m[p] = -INFINITY;
                l[p] = 0.0;
            }
            /* per-partition states */
            for (int p = 0; p < parts; ++p) {
                int t0 = p * partition_tokens;
                int t1 = t0 + partition_tokens < n ? t0 + partition_tokens : n;
                for (int t = t0; t < t1; ++t) {
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += qd[d] * K[(size_t)t * head_dim + d];
                    double s = (double)scale * dot;
                    if (s > m[p])
                        m[p] = s;
                }
                for (int t = t0; t < t1; ++t) {
                    double dot = 0.0;
                    for (int d = 0; d < head_dim; ++d)
                        dot += qd[d] * K[(size_t)t * head_dim + d];
                    double w = exp((double)scale * dot - m[p]);
                    l[p] += w;
                    for (int d = 0; d < head_dim; ++d)
                        a[(size_t)p * head_dim + d] += w * V[(size_t)t * head_dim + d];
                }
            }
            /* merge of the partial results */
            double *o = out + ((size_t)b * num_q_heads + h) * head_dim;
            for (int d = 0; d < head_dim; ++d)
                o[d] = 0.0;
            if (parts > 0) {
                double M = -INFINITY;
                for (int p = 0; p < parts; ++p)
                    if (m[p] > M)
                        M = m[p];
                double L = 0.0;
                for (int p = 0; p < parts; ++p)
                    L += exp(m[p] - M) * l[p];
                for (int p = 0; p < parts; ++p) {
                    double c = exp(m[p] - M);
                    for (int d = 0; d < head_dim; ++d)
                        o[d] += c * a[(size_t)p * head_dim + d];
                }
                for (int d = 0; d < head_dim; ++d)
                    o[d] /= L;
            }
            size_t base = ((size_t)b * num_q_heads + h) * max_parts;
            for (int p = 0; p < max_parts; ++p) {
                if (part_m)
                    part_m[base + p] = m[p];
                if (part_l)
                    part_l[base + p] = l[p];
                if (part_acc)
                    for (int d = 0; d < head_dim; ++d)
                        part_acc[(base + p) * head_dim + d] = a[(size_t)p * head_dim + d];
            }
        }
        free(K);
        free(V);
        free(qd);
        free(m);
        free(l);
        free(a);
    }
    (void)nthreads;
    return status;
}

/* Threads the OpenMP runtime would use for num_threads = 0. */
/* Swap: copy whole blocks (every KV head, every slot, K and V) between two
 * pools of the same block shape -- device blocks out to a host swap space, or
 * back ("08. PagedAttention：把 KV Cache 分页管理", section "分页还顺带解决了什么":
 * a preempted request's blocks move to CPU memory and return later; blocks of
 * one size make the move simple). For each (src, dst) of `block_pairs`
 * ([num_pairs][2]): dst_pool[dst] = src_pool[src], in pair order. */
int oracle_swap_blocks(uint16_t *dst_k, uint16_t *dst_v, int dst_blocks, const uint16_t *src_k,
                       const uint16_t *src_v, int src_blocks, const int64_t *block_pairs,
                       int num_pairs, int num_kv_heads, int block_size, int head_dim)
{
    size_t block_elems = (size_t)num_kv_heads * block_size * head_dim;
    for (int p = 0; p < num_pairs; ++p) {
        int64_t src = block_pairs[2 * p], dst = block_pairs[2 * p + 1];
        if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks)
            return ORC_BAD_BLOCK;
        for (size_t i = 0; i < block_elems; ++i) {
            dst_k[(size_t)dst * block_elems + i] = src_k[(size_t)src * block_elems + i];
            dst_v[(size_t)dst * block_elems + i] = src_v[(size_t)src * block_elems + i];
        }
    }
    return ORC_OK;
}

/* Sliding-window decode ("PagedAttention 核心思想解析", section 5.2: blocks
 * that fall out of the window are reclaimed). Each sequence attends only to
 * its last `window` positions, [lo, n) with lo = max(0, n - window); window
 * <= 0 means no window (all n positions). Only the positions in [lo, n) are
 * looked up, so table entries of blocks wholly before lo may hold anything
 * (a freed block's entry). Same arguments and output as oracle_decode. */
static int gather_span(double *dst, const uint16_t *pool, const int32_t *table_row, int lo,
                       int n, int kv_head, int num_blocks, int num_kv_heads, int block_size,
                       int head_dim, int dtype)
{
    for (int t = lo; t < n; ++t) {
        int64_t slot = oracle_slot(table_row, t, block_size);
        int64_t block = slot / block_size;
        int offset = (int)(slot % block_size);
        if (block < 0 || block >= num_blocks)
            return ORC_BAD_BLOCK;
        for (int d = 0; d < head_dim; ++d)
            dst[(size_t)(t - lo) * head_dim + d] =
                widen(pool[pool_index(block, kv_head, offset, d, num_kv_heads, block_size,
                                      head_dim)], dtype);
    }
    return ORC_OK;
}

int oracle_decode_window(double *out, const uint16_t *q, const uint16_t *k_cache,
                         const uint16_t *v_cache, const int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *context_lens, int num_seqs,
                         int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                         int num_blocks, float scale, int dtype, int window, int num_threads)
{
    int rc = check_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                          num_blocks, max_blocks_per_seq);
    if (rc)
        return rc;
    for (int b = 0; b < num_seqs; ++b)
        if (context_lens[b] < 0 || context_lens[b] > max_blocks_per_seq * block_size)
            return ORC_BAD_ARG;
    int group = num_q_heads / num_kv_heads;
    int nthreads = set_threads(num_threads);
    int status = ORC_OK;
    long long units = (long long)num_seqs * num_q_heads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (long long u = 0; u < units; ++u) {
        int b = (int)(u / num_q_heads), h = (int)(u % num_q_heads);
        int n = context_lens[b];
        int lo = (window > 0 && n > window) ? n - window : 0;
        int m = n - lo;
        int g = h / group;
        double *K = malloc(sizeof(double) * ((size_t)m * head_dim + 1));
        double *V = malloc(sizeof(double) * ((size_t)m * head_dim + 1));
        double *s = malloc(sizeof(double) * ((size_t)m + 1));
        double *qd = malloc(sizeof(double) * (size_t)head_dim);
        const int32_t *row = block_tables + (size_t)b * max_blocks_per_seq;
        int r1 = gather_span(K, k_cache, row, lo, n, g, num_blocks, num_kv_heads, block_size,
                             head_dim, dtype);
        int r2 = gather_span(V, v_cache, row, lo, n, g, num_blocks, num_kv_heads, block_size,
                             head_dim, dtype);
        if (r1 || r2) {
#ifdef _OPENMP
#pragma omp critical
#endif
            status = ORC_BAD_BLOCK;
        } else {
            for (int d = 0; d < head_dim; ++d)
                qd[d] = widen(q[((size_t)b * num_q_heads + h) * head_dim + d], dtype);
            attend_rows(out + ((size_t)b * num_q_heads + h) * head_dim, qd, K, V, m, head_dim,
                        (double)scale, s);
        }
        free(K);
        free(V);
        free(s);
        free(qd);
    }
    (void)nthreads;
    return status;
}

/* Paged attention for several query tokens per sequence (prefill, or a chunk
 * of one): "PagedAttention 核心思想解析", section 2.2 -- the rows of Q are cut
 * into blocks, each scored against the sequence's K/V blocks found through the
 * block table, the partial results merged by position. Sequence b holds
 * n = context_lens[b] positions; its query tokens are rows q_start[b] ..
 * q_start[b+1]-1 of q and are its last m = q_start[b+1] - q_start[b]
 * positions, n-m .. n-1 (their K/V already in the pool). The token at position
 * p attends to positions [lo, p] with lo = max(0, p + 1 - window) when
 * window > 0, else lo = 0: a token sees itself and earlier positions only.
 * out: double [T][num_q_heads][head_dim], T = q_start[num_seqs]. */
int oracle_prefill(double *out, const uint16_t *q, const uint16_t *k_cache,
                   const uint16_t *v_cache, const int32_t *block_tables, int max_blocks_per_seq,
                   const int32_t *context_lens, const int32_t *q_start, int num_seqs,
                   int num_q_heads, int num_kv_heads, int head_dim, int block_size,
                   int num_blocks, float scale, int dtype, int window, int num_threads)
{
    int rc = check_shapes(num_seqs, num_q_heads, num_kv_heads, head_dim, block_size,
                          num_blocks, max_blocks_per_seq);
    if (rc)
        return rc;
    if (q_start[0] != 0)
        return ORC_BAD_ARG;
    for (int b = 0; b < num_seqs; ++b) {
        int m = q_start[b + 1] - q_start[b];
        if (m < 0 || m > context_lens[b] || context_lens[b] > max_blocks_per_seq * block_size)
            return ORC_BAD_ARG;
    }
    int group = num_q_heads / num_kv_heads;
    int nthreads = set_threads(num_threads);
    int status = ORC_OK;
    long long units = (long long)q_start[num_seqs] * num_q_heads;
#ifdef _OPENMP
#pragma omp parallel for schedule(dynamic, 1) num_threads(nthreads)
#endif
    for (long long u = 0; u < units; ++u) {
        int tok = (int)(u / num_q_heads), h = (int)(u % num_q_heads);
        int b = 0;
        while (q_start[b + 1] <= tok)
            ++b;
        int n = context_lens[b];
        int m = q_start[b + 1] - q_start[b];
        int p = n - m + (tok - q_start[b]);           /* this token's position */
        int lo = (window > 0 && p + 1 > window) ? p + 1 - window : 0;
        int cnt = p + 1 - lo;
        int g = h / group;
        double *K = malloc(sizeof(double) * ((size_t)cnt * head_dim + 1));
        double *V = malloc(sizeof(double) * ((size_t)cnt * head_dim + 1));
        double *sc = malloc(sizeof(double) * ((size_t)cnt + 1));
        double *qd = malloc(sizeof(double) * (size_t)head_dim);
        const int32_t *row = block_tables + (size_t)b * max_blocks_per_seq;
        int r1 = gather_span(K, k_cache, row, lo, p + 1, g, num_blocks, num_kv_heads, block_size,
                             head_dim, dtype);
        int r2 = gather_span(V, v_cache, row, lo, p + 1, g, num_blocks, num_kv_heads, block_size,
                             head_dim, dtype);
        if (r1 || r2) {
#ifdef _OPENMP
#pragma omp critical
#endif
            status = ORC_BAD_BLOCK;
        } else {
            for (int d = 0; d < head_dim; ++d)
                qd[d] = widen(q[((size_t)tok * num_q_heads + h) * head_dim + d], dtype);
            attend_rows(out + ((size_t)tok * num_q_heads + h) * head_dim, qd, K, V, cnt,
                        head_dim, (double)scale, sc);
        }
        free(K);
        free(V);
        free(sc);
        free(qd);
    }
    (void)nthreads;
    return status;
}

int oracle_max_threads(void)
{
    return set_threads(0);
}

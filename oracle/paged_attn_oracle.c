/*
 * Float64 CPU oracle for one-token paged decode attention and the KV append.
 *
 * TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark load this code.  It shares nothing with the
 * CUDA library (no header, helper, table or constant) and is written to be
 * read against the pages, not to be fast:
 *
 *   - every input value is widened to double (exact for fp32 and bf16);
 *   - the address translation is the chain the BareLLM README gives in its
 *     cache section: position -> logical block (pos // block_size) ->
 *     block_table -> physical block -> K/V, over storage shaped
 *     [physical_blocks, block_size, kv_heads, head_dim] (NHD order,
 *     BareLLM README, "Cache layers" bullets);
 *   - attention is softmax(q . K^T * scale) . V over the request's own
 *     context (BareLLM README feature list: one-token batched decode with
 *     unequal request lengths; MHA/GQA/MQA), written with straight sums:
 *     all scores, then their maximum, then the weights and the two sums.
 *     It does not use the running-max (online softmax) form the MinivLLM
 *     review and the LLAISYS self-attention bullet describe, so that the
 *     GPU's algorithm is checked against the definition, not against itself;
 *   - the grouped-query head map is contiguous: query head h reads KV head
 *     h / (Hq / Hkv), the "repeat each KV head Hq/Hkv times" form of GQA
 *     (MQA is Hkv = 1, MHA is Hkv = Hq);
 *   - chunked prefill (oracle_prefill) applies the same definition to every
 *     new token of a request over the positions up to its own (causal);
 *   - the partitioned form (oracle_decode_partitioned) splits each context
 *     into fixed token partitions, keeps (max, sum of weights, weighted sum
 *     of V) per partition and combines them by log-sum-exp; it exists only
 *     to pin that combination against the unsplit definition.
 *
 * Parallelism: OpenMP over independent (request, query head) pairs; the
 * arithmetic inside one pair is sequential and in a fixed order.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F32 0
#define ORACLE_BF16 1
#define ORACLE_F16 2

typedef struct {
    const void *q;              /* [B, Hq, D] */
    const void *k_cache;        /* [num_blocks, block_size, Hkv, D] */
    const void *v_cache;        /* [num_blocks, block_size, Hkv, D] */
    const int32_t *block_tables;/* [B, max_blocks_per_seq] */
    const int32_t *context_lens;/* [B] */
    double scale;
    int32_t B, Hq, Hkv, D;
    int32_t block_size, num_blocks, max_blocks_per_seq;
    int32_t dtype;              /* ORACLE_F32, ORACLE_BF16 or ORACLE_F16 */
} oracle_problem;

/* IEEE 754 binary16 -> double (exact): sign, 5 exponent bits (bias 15),
 * 10 fraction bits; exponent 0 is subnormal, 31 is infinity / NaN. */
static double half_to_double(uint16_t h)
{
    int sign = h >> 15, e = (h >> 10) & 0x1F, f = h & 0x3FF;
    double v;
    if (e == 0)
        v = ldexp((double)f, -24);
    else if (e == 31)
        v = f ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + f), e - 25);
    return sign ? -v : v;
}

/* One stored value, widened to double.  bf16 is the upper half of an IEEE
 * binary32, so shifting its 16 bits up gives the float exactly. */
static double value_at(const void *base, int64_t i, int dtype)
{
    if (dtype == ORACLE_F32)
        return (double)((const float *)base)[i];
    if (dtype == ORACLE_F16)
        return half_to_double(((const uint16_t *)base)[i]);
    uint32_t bits = ((uint32_t)((const uint16_t *)base)[i]) << 16;
    float f;
    memcpy(&f, &bits, sizeof f);
    return (double)f;
}

static int check_problem(const oracle_problem *p)
{
    if (!p || !p->q || !p->k_cache || !p->v_cache || !p->block_tables || !p->context_lens)
        return -1;
    if (p->B < 0 || p->Hq <= 0 || p->Hkv <= 0 || p->D <= 0 || p->Hq % p->Hkv != 0)
        return -2;
    if (p->block_size <= 0 || p->num_blocks < 0 || p->max_blocks_per_seq < 0)
        return -3;
    if (p->dtype != ORACLE_F32 && p->dtype != ORACLE_BF16 && p->dtype != ORACLE_F16)
        return -4;
    for (int b = 0; b < p->B; ++b) {
        int32_t L = p->context_lens[b];
        if (L < 0 || (int64_t)L > (int64_t)p->max_blocks_per_seq * p->block_size)
            return -5;
        int32_t nblk = (L + p->block_size - 1) / p->block_size;
        for (int j = 0; j < nblk; ++j) {
            int32_t phys = p->block_tables[(int64_t)b * p->max_blocks_per_seq + j];
            if (phys < 0 || phys >= p->num_blocks)
                return -6;
        }
    }
    return 0;
}

/* Flat element index of K/V element d of token t (of request b) for KV head g:
 * logical block t / block_size, offset t % block_size, physical block from
 * the request's block table, then the NHD layout of the pool. */
static int64_t kv_index(const oracle_problem *p, int b, int t, int g, int d)
{
    int32_t logical_block = t / p->block_size;
    int32_t offset = t % p->block_size;
    int32_t phys = p->block_tables[(int64_t)b * p->max_blocks_per_seq + logical_block];
    return (((int64_t)phys * p->block_size + offset) * p->Hkv + g) * p->D + d;
}

/* Score of token t for query head h of request b: scale * sum_d q[d] K[t][d]. */
static double score(const oracle_problem *p, int b, int h, int t)
{
    int g = h / (p->Hq / p->Hkv);
    double dot = 0.0;
    for (int d = 0; d < p->D; ++d) {
        double qd = value_at(p->q, ((int64_t)b * p->Hq + h) * p->D + d, p->dtype);
        double kd = value_at(p->k_cache, kv_index(p, b, t, g, d), p->dtype);
        dot += qd * kd;
    }
    return p->scale * dot;
}

/* out[0..D) = softmax over t < L of the scores, applied to V.  L = 0 gives 0. */
static void attend_one(const oracle_problem *p, int b, int h, double *s, double *out)
{
    int L = p->context_lens[b];
    int g = h / (p->Hq / p->Hkv);
    for (int d = 0; d < p->D; ++d)
        out[d] = 0.0;
    if (L == 0)
        return;
    for (int t = 0; t < L; ++t)
        s[t] = score(p, b, h, t);
    double m = s[0];
    for (int t = 1; t < L; ++t)
        if (s[t] > m)
            m = s[t];
    double den = 0.0;
    for (int t = 0; t < L; ++t) {
        double w = exp(s[t] - m);
        den += w;
        for (int d = 0; d < p->D; ++d)
            out[d] += w * value_at(p->v_cache, kv_index(p, b, t, g, d), p->dtype);
    }
    for (int d = 0; d < p->D; ++d)
        out[d] /= den;
}

static int max_context(const oracle_problem *p)
{
    int m = 1;
    for (int b = 0; b < p->B; ++b)
        if (p->context_lens[b] > m)
            m = p->context_lens[b];
    return m;
}

/* Full decode: out[B, Hq, D] in double.  nthreads <= 0 uses OpenMP's default.
 * Returns 0, or a negative code for a malformed problem (nothing is read out
 * of bounds). */
int oracle_decode(const oracle_problem *p, double *out, int nthreads)
{
    int rc = check_problem(p);
    if (rc)
        return rc;
    int64_t pairs = (int64_t)p->B * p->Hq;
    int Lmax = max_context(p);
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : omp_get_max_threads())
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Lmax);
        if (!s) {
#pragma omp atomic write
            err = -7;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < pairs; ++i) {
            if (s)
                attend_one(p, (int)(i / p->Hq), (int)(i % p->Hq), s, out + i * p->D);
        }
        free(s);
    }
    return err;
}

/* Decode for a list of (b, h) pairs only (pairs[2*i], pairs[2*i+1]);
 * out[npairs, D].  Used to check sampled outputs of large batches. */
int oracle_decode_pairs(const oracle_problem *p, const int32_t *pairs, int npairs, double *out,
                        int nthreads)
{
    int rc = check_problem(p);
    if (rc)
        return rc;
    for (int i = 0; i < npairs; ++i)
        if (pairs[2 * i] < 0 || pairs[2 * i] >= p->B || pairs[2 * i + 1] < 0 || pairs[2 * i + 1] >= p->Hq)
            return -8;
    int Lmax = max_context(p);
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : omp_get_max_threads())
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Lmax);
        if (!s) {
#pragma omp atomic write
            err = -7;
        }
#pragma omp for schedule(dynamic, 1)
        for (int i = 0; i < npairs; ++i) {
            if (s)
                attend_one(p, pairs[2 * i], pairs[2 * i + 1], s, out + (int64_t)i * p->D);
        }
        free(s);
    }
    return err;
}

/* Partitioned form: for each (b, h) the context is cut into partitions of
 * partition_tokens tokens.  Partition i keeps
 *     m_i = max_t s_t,  l_i = sum_t exp(s_t - m_i),  o_i = sum_t exp(s_t - m_i) V_t
 * and the partitions are combined by log-sum-exp:
 *     M = max_i m_i,  out = sum_i exp(m_i - M) o_i / sum_i exp(m_i - M) l_i.
 * A partition with no tokens contributes nothing. */
int oracle_decode_partitioned(const oracle_problem *p, int partition_tokens, double *out, int nthreads)
{
    int rc = check_problem(p);
    if (rc)
        return rc;
    if (partition_tokens <= 0)
        return -9;
    int64_t pairs = (int64_t)p->B * p->Hq;
    int Lmax = max_context(p);
    int max_parts = (Lmax + partition_tokens - 1) / partition_tokens;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : omp_get_max_threads())
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Lmax);
        double *pm = (double *)malloc(sizeof(double) * (size_t)max_parts);
        double *pl = (double *)malloc(sizeof(double) * (size_t)max_parts);
        double *po = (double *)malloc(sizeof(double) * (size_t)max_parts * (size_t)p->D);
        if (!s || !pm || !pl || !po) {
#pragma omp atomic write
            err = -7;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < pairs; ++i) {
            if (!(s && pm && pl && po))
                continue;
            int b = (int)(i / p->Hq), h = (int)(i % p->Hq);
            int g = h / (p->Hq / p->Hkv);
            int L = p->context_lens[b];
            double *o = out + i * p->D;
            for (int d = 0; d < p->D; ++d)
                o[d] = 0.0;
            if (L == 0)
                continue;
            int nparts = (L + partition_tokens - 1) / partition_tokens;
            for (int part = 0; part < nparts; ++part) {
                int t0 = part * partition_tokens;
                int t1 = t0 + partition_tokens < L ? t0 + partition_tokens : L;
                for (int t = t0; t < t1; ++t)
                    s[t] = score(p, b, h, t);
                double m = s[t0];
                for (int t = t0 + 1; t < t1; ++t)
                    if (s[t] > m)
                        m = s[t];
                double l = 0.0;
                double *oi = po + (size_t)part * p->D;
                for (int d = 0; d < p->D; ++d)
                    oi[d] = 0.0;
                for (int t = t0; t < t1; ++t) {
                    double w = exp(s[t] - m);
                    l += w;
                    for (int d = 0; d < p->D; ++d)
                        oi[d] += w * value_at(p->v_cache, kv_index(p, b, t, g, d), p->dtype);
                }
                pm[part] = m;
                pl[part] = l;
            }
            double M = pm[0];
            for (int part = 1; part < nparts; ++part)
                if (pm[part] > M)
                    M = pm[part];
            double den = 0.0;
            for (int part = 0; part < nparts; ++part) {
                double c = exp(pm[part] - M);
                den += c * pl[part];
                for (int d = 0; d < p->D; ++d)
                    o[d] += c * po[(size_t)part * p->D + d];
            }
            for (int d = 0; d < p->D; ++d)
                o[d] /= den;
        }
        free(s);
        free(pm);
        free(pl);
        free(po);
    }
    return err;
}

/* Chunked prefill: the step before decode, in which a request's new tokens
 * attend to its cached history and to each other, causally (the MinivLLM
 * review's prefill path, read over the paged cache).  Request b owns rows
 * query_start[b] .. query_start[b+1]-1 of q and of out: n_b new tokens, the
 * last n_b of its context_lens[b] positions, whose K/V are already in the
 * cache (written by the append, one slot per token).  New token j sits at
 * position pos = context_lens[b] - n_b + j and attends to positions
 * 0 .. pos: the decode definition above applied to that prefix, with q row
 * query_start[b] + j. */
static double score_prefill(const oracle_problem *p, int64_t row, int b, int h, int t)
{
    int g = h / (p->Hq / p->Hkv);
    double dot = 0.0;
    for (int d = 0; d < p->D; ++d) {
        double qd = value_at(p->q, (row * p->Hq + h) * p->D + d, p->dtype);
        double kd = value_at(p->k_cache, kv_index(p, b, t, g, d), p->dtype);
        dot += qd * kd;
    }
    return p->scale * dot;
}

static void attend_prefill(const oracle_problem *p, int64_t row, int b, int h, int visible, double *s,
                           double *out)
{
    int g = h / (p->Hq / p->Hkv);
    for (int d = 0; d < p->D; ++d)
        out[d] = 0.0;
    if (visible <= 0)
        return;
    for (int t = 0; t < visible; ++t)
        s[t] = score_prefill(p, row, b, h, t);
    double m = s[0];
    for (int t = 1; t < visible; ++t)
        if (s[t] > m)
            m = s[t];
    double den = 0.0;
    for (int t = 0; t < visible; ++t) {
        double w = exp(s[t] - m);
        den += w;
        for (int d = 0; d < p->D; ++d)
            out[d] += w * value_at(p->v_cache, kv_index(p, b, t, g, d), p->dtype);
    }
    for (int d = 0; d < p->D; ++d)
        out[d] /= den;
}

/* out[T, Hq, D] for the T = query_start[B] new tokens.  Returns 0, or a
 * negative code for a malformed problem (query_start not starting at 0,
 * decreasing, or giving a request more new tokens than its context holds). */
int oracle_prefill(const oracle_problem *p, const int32_t *query_start, double *out, int nthreads)
{
    int rc = check_problem(p);
    if (rc)
        return rc;
    if (!query_start || query_start[0] != 0)
        return -10;
    for (int b = 0; b < p->B; ++b) {
        int32_t n = query_start[b + 1] - query_start[b];
        if (n < 0 || n > p->context_lens[b])
            return -10;
    }
    int64_t T = query_start[p->B];
    int64_t pairs = T * p->Hq;
    int Lmax = max_context(p);
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : omp_get_max_threads())
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Lmax);
        if (!s) {
#pragma omp atomic write
            err = -7;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < pairs; ++i) {
            if (!s)
                continue;
            int64_t row = i / p->Hq;
            int h = (int)(i % p->Hq);
            int lo = 0, hi = p->B;  /* request owning the row: query_start[b] <= row < query_start[b+1] */
            while (hi - lo > 1) {
                int mid = (lo + hi) / 2;
                if (query_start[mid] <= row)
                    lo = mid;
                else
                    hi = mid;
            }
            int b = lo;
            int n = query_start[b + 1] - query_start[b];
            int pos = p->context_lens[b] - n + (int)(row - query_start[b]);
            attend_prefill(p, row, b, h, pos + 1, s, out + i * p->D);
        }
        free(s);
    }
    return err;
}

/* oracle_prefill for the listed rows only (all heads): out[nrows, Hq, D].
 * Used to check sampled rows of large prefill steps. */
int oracle_prefill_rows(const oracle_problem *p, const int32_t *query_start, const int64_t *rows, int nrows,
                        double *out, int nthreads)
{
    int rc = check_problem(p);
    if (rc)
        return rc;
    if (!query_start || query_start[0] != 0)
        return -10;
    for (int b = 0; b < p->B; ++b) {
        int32_t n = query_start[b + 1] - query_start[b];
        if (n < 0 || n > p->context_lens[b])
            return -10;
    }
    for (int i = 0; i < nrows; ++i)
        if (rows[i] < 0 || rows[i] >= query_start[p->B])
            return -11;
    int Lmax = max_context(p);
    int64_t pairs = (int64_t)nrows * p->Hq;
    int err = 0;
#pragma omp parallel num_threads(nthreads > 0 ? nthreads : omp_get_max_threads())
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)Lmax);
        if (!s) {
#pragma omp atomic write
            err = -7;
        }
#pragma omp for schedule(dynamic, 1)
        for (int64_t i = 0; i < pairs; ++i) {
            if (!s)
                continue;
            int64_t row = rows[i / p->Hq];
            int h = (int)(i % p->Hq);
            int lo = 0, hi = p->B;
            while (hi - lo > 1) {
                int mid = (lo + hi) / 2;
                if (query_start[mid] <= row)
                    lo = mid;
                else
                    hi = mid;
            }
            int b = lo;
            int n = query_start[b + 1] - query_start[b];
            int pos = p->context_lens[b] - n + (int)(row - query_start[b]);
            attend_prefill(p, row, b, h, pos + 1, s, out + i * p->D);
        }
        free(s);
    }
    return err;
}

/* KV append: for each request i with slot s = slot_mapping[i] >= 0, copy the
 * new token's K (all KV heads) into block s / block_size, offset
 * s % block_size, and the same for V (the BareLLM README's "logical-to-
 * physical writes" of PagedKVCache).  A byte copy, so the result is exact in
 * either dtype.  Requests with s < 0 are skipped.  Returns the number of
 * tokens written, or a negative code if a slot lies outside the pool (then
 * nothing is written). */
int oracle_kv_append(const void *k_new, const void *v_new, const int32_t *slot_mapping, void *k_cache,
                     void *v_cache, int B, int Hkv, int D, int block_size, int num_blocks, int dtype)
{
    if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache || B < 0 || Hkv <= 0 || D <= 0 ||
        block_size <= 0 || num_blocks < 0)
        return -1;
    size_t elem = dtype == ORACLE_F32 ? 4 : 2;
    size_t token_bytes = (size_t)Hkv * (size_t)D * elem; /* one token, all KV heads, NHD */
    for (int i = 0; i < B; ++i)
        if ((int64_t)slot_mapping[i] >= (int64_t)num_blocks * block_size)
            return -2;
    int written = 0;
    for (int i = 0; i < B; ++i) {
        int32_t s = slot_mapping[i];
        if (s < 0)
            continue;
        int64_t block = s / block_size;
        int64_t offset = s % block_size;
        size_t dst = (size_t)(block * block_size + offset) * token_bytes;
        memcpy((char *)k_cache + dst, (const char *)k_new + (size_t)i * token_bytes, token_bytes);
        memcpy((char *)v_cache + dst, (const char *)v_new + (size_t)i * token_bytes, token_bytes);
        ++written;
    }
    return written;
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

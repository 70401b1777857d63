/*
 * pa_oracle.c -- plain, slow, float64 CPU oracle for paged-attention decode.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
 * CPU-baseline / reference arm may load this file's library.  It shares no
 * code, header, table or helper with the CUDA library: it has its own bf16
 * decoding, its own block-table walk and its own softmax.
 *
 * What it computes (sources, by page and section):
 *
 *  - gllm PR #116 "feat(backend): sliding-window PagedAttention", section
 *    "What changes": the call is PagedAttention(dst, q, kCache, vCache,
 *    blockTables, seqLens, queryLens, scale, window).  With window > 0 the
 *    token at position p attends to positions p-window+1 .. p only; window 0
 *    keeps unlimited causal attention.  The CPU reference starts each query
 *    token's visible range at max(0, end-window).
 *  - ExecuTorch PR #18759 "SDPA decode perf improvements for
 *    qwen-3.5-35B-A3B", sdpa_decode_splitk docstring: grouped-query heads map
 *    to kv head h // (H_q / H_kv).
 *  - Same ExecuTorch page, review suggestion 5 ("Partial accumulator stores
 *    unscaled acc"): split-K partitions produce partial (max, sum, output)
 *    that a reduce step rescales and merges.  The split mode below follows
 *    that log-sum-exp merge.
 *
 * Readings taken where the pages are silent (each is also listed in the
 * design notes of the repository):
 *  - seqLens[b] counts every cached token of row b, including its
 *    queryLens[b] new tokens, which sit at positions S-L .. S-1 and are
 *    causal among themselves.  So query token i sits at p = S - L + i and
 *    sees [lo, p+1) with lo = window > 0 ? max(0, p+1-window) : 0.
 *  - Cache layout [num_blocks][H_kv][block_size][head_dim]; token t of row b
 *    lives in physical block blockTables[b][t / block_size], slot
 *    t % block_size.
 *  - q and the output are packed [sum(queryLens)][H_q][head_dim], rows in
 *    batch order.
 *  - scale is used exactly as passed.
 *  - windows[b], when given, overrides the scalar window for row b.
 *
 * FP8 operands (aiter PR #2914 "Pa gluon swa mtp opt", review of
 * pa_decode_gluon's query_scale / key_scale / value_scale): an FP8 query or
 * FP8 caches hold e4m3 codes, and an element's value is its code's number
 * times the tensor's scale.
 *
 * Arithmetic: inputs are bf16 bit patterns, widened exactly to double; every
 * sum, exponential and division is done in double, in the two-pass form of
 * the definition (exact maximum first, then the normalised sum).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_OK 0
#define ORACLE_EINVAL -1

/* bf16 bit pattern -> double.  A bf16 value is the upper half of an IEEE
 * binary32, so the widening is exact. */
static double bf16_bits_to_double(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* FP8 e4m3 bit pattern -> double: sign, 4-bit exponent (bias 7), 3-bit
 * mantissa; exponent 0 is subnormal (m/8 * 2^-6); the two codes with every
 * exponent and mantissa bit set are NaN; there is no infinity. */
static double e4m3_bits_to_double(uint8_t x)
{
    int sign = x >> 7, e = (x >> 3) & 15, m = x & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m / 8.0, -6);
    else v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -v : v;
}

typedef struct {
    const void *q;         /* bf16 (uint16) or, with q_fp8, e4m3 (uint8) elements */
    const void *kc, *vc;   /* bf16 (uint16) or, with kv_fp8, e4m3 (uint8) elements */
    const int32_t *block_tables, *seq_lens, *query_lens, *windows;
    int window;
    double scale;
    int batch, hq, hkv, d, bs, num_blocks, mbps;
    int kv_fp8;            /* caches hold e4m3 codes; value = code * k_scale (v_scale) */
    double k_scale, v_scale;
    int q_fp8;             /* q holds e4m3 codes; value = code * q_scale */
    double q_scale;
} problem;

/* Element idx of a cache as a double (dequantised for FP8 caches). */
static double kv_value(const problem *pr, const void *cache, size_t idx, double s)
{
    if (pr->kv_fp8) return s * e4m3_bits_to_double(((const uint8_t *)cache)[idx]);
    return bf16_bits_to_double(((const uint16_t *)cache)[idx]);
}

/* Element idx of q as a double (dequantised for an FP8 query). */
static double q_value(const problem *pr, size_t idx)
{
    if (pr->q_fp8) return pr->q_scale * e4m3_bits_to_double(((const uint8_t *)pr->q)[idx]);
    return bf16_bits_to_double(((const uint16_t *)pr->q)[idx]);
}

/* Exported for the tests: decodes n e4m3 codes. */
void oracle_e4m3_decode(double *out, const uint8_t *codes, int n)
{
    for (int i = 0; i < n; ++i) out[i] = e4m3_bits_to_double(codes[i]);
}

static int row_window(const problem *pr, int b)
{
    return pr->windows ? pr->windows[b] : pr->window;
}

/* Visible range of query token i of a row with seq_len S and query_len L:
 * the token sits at p = S - L + i and sees [lo, p + 1). */
int oracle_visible_range(int seq_len, int query_len, int i, int window,
                         int *lo, int *hi)
{
    if (query_len < 0 || seq_len < 0 || query_len > seq_len || window < 0 ||
        i < 0 || i >= query_len)
        return ORACLE_EINVAL;
    int p = seq_len - query_len + i;
    int end = p + 1;
    int start = 0;
    if (window > 0) {
        start = end - window;
        if (start < 0) start = 0;
    }
    *lo = start;
    *hi = end;
    return ORACLE_OK;
}

/* Visible ranges of every query token, packed in batch order. */
int oracle_visible_ranges(int32_t *lo, int32_t *hi, const int32_t *seq_lens,
                          const int32_t *query_lens, const int32_t *windows,
                          int window, int batch)
{
    int n = 0;
    for (int b = 0; b < batch; ++b) {
        int w = windows ? windows[b] : window;
        for (int i = 0; i < query_lens[b]; ++i) {
            int l, h;
            if (oracle_visible_range(seq_lens[b], query_lens[b], i, w, &l, &h))
                return ORACLE_EINVAL;
            lo[n] = l;
            hi[n] = h;
            ++n;
        }
    }
    return n;
}

/* Leading KV blocks of each row that no query token of this call, nor any
 * later token of the row (later tokens sit at larger positions, so their
 * windows start no earlier), can see: the blocks that end at or before the
 * lowest visible position of the row's tokens.  Window 0 sees everything, so
 * nothing is dead.  gllm PR #116 "feat(backend): sliding-window
 * PagedAttention", "What changes": the cache keeps every position; freeing
 * blocks a window can no longer reach is a separate step. */
int oracle_unreachable_blocks(int32_t *count, const int32_t *seq_lens,
                              const int32_t *query_lens, const int32_t *windows,
                              int window, int bs, int batch)
{
    for (int b = 0; b < batch; ++b) {
        int w = windows ? windows[b] : window;
        count[b] = 0;
        if (query_lens[b] <= 0 || w == 0) continue;
        int lowest = seq_lens[b];
        for (int i = 0; i < query_lens[b]; ++i) {
            int lo, hi;
            if (oracle_visible_range(seq_lens[b], query_lens[b], i, w, &lo, &hi))
                return ORACLE_EINVAL;
            if (lo < lowest) lowest = lo;
        }
        count[b] = lowest / bs;
    }
    return ORACLE_OK;
}

static int validate(const problem *pr)
{
    if (pr->batch < 0 || pr->hq <= 0 || pr->hkv <= 0 || pr->d <= 0 ||
        pr->bs <= 0 || pr->num_blocks <= 0 || pr->mbps <= 0)
        return ORACLE_EINVAL;
    if (pr->hq % pr->hkv != 0) return ORACLE_EINVAL;
    if (pr->window < 0) return ORACLE_EINVAL;
    for (int b = 0; b < pr->batch; ++b) {
        int S = pr->seq_lens[b], L = pr->query_lens[b];
        if (L < 0 || S < 0 || L > S) return ORACLE_EINVAL;
        if (row_window(pr, b) < 0) return ORACLE_EINVAL;
        if (L == 0) continue;
        int nblk = (S + pr->bs - 1) / pr->bs;
        if (nblk > pr->mbps) return ORACLE_EINVAL;
        for (int j = 0; j < nblk; ++j) {
            int phys = pr->block_tables[(size_t)b * pr->mbps + j];
            if (phys < 0 || phys >= pr->num_blocks) return ORACLE_EINVAL;
        }
    }
    return ORACLE_OK;
}

/* Address of element d of token t of kv head g of row b in a cache. */
static size_t cache_index(const problem *pr, int b, int g, int t)
{
    int phys = pr->block_tables[(size_t)b * pr->mbps + t / pr->bs];
    int slot = t % pr->bs;
    return (((size_t)phys * pr->hkv + g) * pr->bs + slot) * (size_t)pr->d;
}

/* Score of query (row b, token i, head h) against cached token t:
 * scale * sum_d q[d] * k_t[d]. */
static double score(const problem *pr, size_t qrow, int b, int g, int t)
{
    const size_t k = cache_index(pr, b, g, t);
    double acc = 0.0;
    for (int x = 0; x < pr->d; ++x)
        acc += q_value(pr, qrow + x) * kv_value(pr, pr->kc, k + x, pr->k_scale);
    return pr->scale * acc;
}

static size_t qrow_offset(const problem *pr, int b, int i, int h)
{
    size_t tok = 0;
    for (int bb = 0; bb < b; ++bb) tok += (size_t)pr->query_lens[bb];
    tok += (size_t)i;
    return (tok * pr->hq + h) * (size_t)pr->d;
}

/* Softmax attention of one query over the cached tokens [t0, t1): writes the
 * normalised output (length d) and returns its log-sum-exp
 * M + log(sum exp(s - M)).  An empty range gives lse = -inf and a zero
 * output: a partition that sees nothing contributes nothing.  When w is not
 * NULL it receives the weights of [t0, t1). */
static double attend_range(const problem *pr, int b, int i, int h, int t0,
                           int t1, double *out, double *w)
{
    int g = h / (pr->hq / pr->hkv);
    const size_t qrow = qrow_offset(pr, b, i, h);
    for (int x = 0; x < pr->d; ++x) out[x] = 0.0;
    if (t1 <= t0) return -INFINITY;

    int n = t1 - t0;
    double *s = (double *)malloc(sizeof(double) * (size_t)n);
    if (!s) return NAN;
    /* pass 1: scores and their exact maximum */
    double m = -INFINITY;
    for (int t = t0; t < t1; ++t) {
        s[t - t0] = score(pr, qrow, b, g, t);
        if (s[t - t0] > m) m = s[t - t0];
    }
    /* pass 2: normaliser */
    double z = 0.0;
    for (int j = 0; j < n; ++j) z += exp(s[j] - m);
    /* weights and the weighted sum of values */
    for (int t = t0; t < t1; ++t) {
        double a = exp(s[t - t0] - m) / z;
        if (w) w[t - t0] = a;
        const size_t v = cache_index(pr, b, g, t);
        for (int x = 0; x < pr->d; ++x) out[x] += a * kv_value(pr, pr->vc, v + x, pr->v_scale);
    }
    free(s);
    return m + log(z);
}

/* Output of one query in split-K form: the row's visible union is cut into
 * `parts` equal chunks (the last one takes the remainder); each chunk yields
 * (lse_p, O_p) over its intersection with this query's range, and the chunks
 * are merged with weights exp(lse_p - max lse). */
static int attend_split(const problem *pr, int b, int i, int h, int parts,
                        double *out)
{
    int S = pr->seq_lens[b], L = pr->query_lens[b];
    int w = row_window(pr, b);
    int lo, hi, ulo, uhi;
    oracle_visible_range(S, L, i, w, &lo, &hi);
    oracle_visible_range(S, L, 0, w, &ulo, &uhi); /* union starts at token 0's lo */
    uhi = S;
    int span = uhi - ulo;
    int chunk = (span + parts - 1) / parts;
    if (chunk < 1) chunk = 1;

    double *lse = (double *)malloc(sizeof(double) * (size_t)parts);
    double *o = (double *)malloc(sizeof(double) * (size_t)parts * pr->d);
    if (!lse || !o) { free(lse); free(o); return ORACLE_EINVAL; }
    double mmax = -INFINITY;
    for (int p = 0; p < parts; ++p) {
        int c0 = ulo + p * chunk, c1 = c0 + chunk;
        if (c1 > uhi) c1 = uhi;
        int a0 = c0 > lo ? c0 : lo, a1 = c1 < hi ? c1 : hi;
        lse[p] = attend_range(pr, b, i, h, a0, a1, o + (size_t)p * pr->d, NULL);
        if (lse[p] > mmax) mmax = lse[p];
    }
    double z = 0.0;
    for (int x = 0; x < pr->d; ++x) out[x] = 0.0;
    for (int p = 0; p < parts; ++p) {
        if (lse[p] == -INFINITY) continue;
        double wt = exp(lse[p] - mmax);
        z += wt;
        for (int x = 0; x < pr->d; ++x) out[x] += wt * o[(size_t)p * pr->d + x];
    }
    for (int x = 0; x < pr->d; ++x) out[x] /= z;
    free(lse);
    free(o);
    return ORACLE_OK;
}

/* One output vector for (b, i, h): direct form when parts == 0, else split. */
static int attend_one(const problem *pr, int b, int i, int h, int parts,
                      double *out, double *w)
{
    if (parts > 0) return attend_split(pr, b, i, h, parts, out);
    int lo, hi;
    if (oracle_visible_range(pr->seq_lens[b], pr->query_lens[b], i,
                             row_window(pr, b), &lo, &hi))
        return ORACLE_EINVAL;
    attend_range(pr, b, i, h, lo, hi, out, w);
    return ORACLE_OK;
}

static void set_threads(int nthreads)
{
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#else
    (void)nthreads;
#endif
}

/* Number of threads the oracle's parallel loops use. */
int oracle_max_threads(int nthreads)
{
#ifdef _OPENMP
    set_threads(nthreads);
    return omp_get_max_threads();
#else
    (void)nthreads;
    return 1;
#endif
}

/* Every output: out is [sum(queryLens)][H_q][head_dim] doubles.
 * parts == 0: direct two-pass softmax; parts > 0: split-K with that many
 * partitions per row, merged by log-sum-exp. */
int oracle_pa_decode(double *out, const void *q, const void *kc,
                     const void *vc, const int32_t *block_tables,
                     const int32_t *seq_lens, const int32_t *query_lens,
                     const int32_t *windows, int window, double scale,
                     int batch, int hq, int hkv, int d, int bs, int num_blocks,
                     int max_blocks_per_seq, int kv_fp8, double k_scale, double v_scale,
                     int q_fp8, double q_scale, int parts, int nthreads)
{
    problem pr = {q, kc, vc, block_tables, seq_lens, query_lens, windows,
                  window, scale, batch, hq, hkv, d, bs, num_blocks,
                  max_blocks_per_seq, kv_fp8, k_scale, v_scale, q_fp8, q_scale};
    if (validate(&pr) || parts < 0) return ORACLE_EINVAL;
    /* list every (b, i, h) with its output slot */
    size_t ntok = 0;
    for (int b = 0; b < batch; ++b) ntok += (size_t)query_lens[b];
    long total = (long)ntok * hq;
    int *bi = (int *)malloc(sizeof(int) * 2 * (ntok ? ntok : 1));
    if (!bi) return ORACLE_EINVAL;
    size_t n = 0;
    for (int b = 0; b < batch; ++b)
        for (int i = 0; i < query_lens[b]; ++i) { bi[2 * n] = b; bi[2 * n + 1] = i; ++n; }
    int err = 0;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (long idx = 0; idx < total; ++idx) {
        long tok = idx / hq;
        int h = (int)(idx % hq);
        err |= attend_one(&pr, bi[2 * tok], bi[2 * tok + 1], h, parts,
                          out + (size_t)idx * d, NULL) != ORACLE_OK;
    }
    free(bi);
    return err ? ORACLE_EINVAL : ORACLE_OK;
}

/* A chosen subset of outputs: sel is [nsel][3] (b, i, h); out is [nsel][d]. */
int oracle_pa_decode_select(double *out, const int32_t *sel, int nsel,
                            const void *q, const void *kc,
                            const void *vc, const int32_t *block_tables,
                            const int32_t *seq_lens, const int32_t *query_lens,
                            const int32_t *windows, int window, double scale,
                            int batch, int hq, int hkv, int d, int bs,
                            int num_blocks, int max_blocks_per_seq, int kv_fp8,
                            double k_scale, double v_scale, int q_fp8,
                            double q_scale, int nthreads)
{
    problem pr = {q, kc, vc, block_tables, seq_lens, query_lens, windows,
                  window, scale, batch, hq, hkv, d, bs, num_blocks,
                  max_blocks_per_seq, kv_fp8, k_scale, v_scale, q_fp8, q_scale};
    if (validate(&pr)) return ORACLE_EINVAL;
    for (int j = 0; j < nsel; ++j) {
        int b = sel[3 * j], i = sel[3 * j + 1], h = sel[3 * j + 2];
        if (b < 0 || b >= batch || i < 0 || i >= query_lens[b] || h < 0 || h >= hq)
            return ORACLE_EINVAL;
    }
    int err = 0;
    set_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
    for (int j = 0; j < nsel; ++j)
        err |= attend_one(&pr, sel[3 * j], sel[3 * j + 1], sel[3 * j + 2], 0,
                          out + (size_t)j * d, NULL) != ORACLE_OK;
    return err ? ORACLE_EINVAL : ORACLE_OK;
}

/* Softmax weights of one query (b, i, h) over every cached position of its
 * row: w is [seq_lens[b]] doubles, zero outside the visible range. */
int oracle_softmax_weights(double *w, int b, int i, int h, const void *q,
                           const void *kc, const void *vc,
                           const int32_t *block_tables, const int32_t *seq_lens,
                           const int32_t *query_lens, const int32_t *windows,
                           int window, double scale, int batch, int hq, int hkv,
                           int d, int bs, int num_blocks, int max_blocks_per_seq,
                           int kv_fp8, double k_scale, double v_scale,
                           int q_fp8, double q_scale)
{
    problem pr = {q, kc, vc, block_tables, seq_lens, query_lens, windows,
                  window, scale, batch, hq, hkv, d, bs, num_blocks,
                  max_blocks_per_seq, kv_fp8, k_scale, v_scale, q_fp8, q_scale};
    if (validate(&pr)) return ORACLE_EINVAL;
    if (b < 0 || b >= batch || i < 0 || i >= query_lens[b] || h < 0 || h >= hq)
        return ORACLE_EINVAL;
    int lo, hi;
    oracle_visible_range(seq_lens[b], query_lens[b], i, row_window(&pr, b), &lo, &hi);
    for (int t = 0; t < seq_lens[b]; ++t) w[t] = 0.0;
    double *out = (double *)malloc(sizeof(double) * (size_t)d);
    if (!out) return ORACLE_EINVAL;
    attend_range(&pr, b, i, h, lo, hi, out, w + lo);
    free(out);
    return ORACLE_OK;
}

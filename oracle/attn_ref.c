/*
 * Oracle: single-query attention over a block-paged KV cache, in fp64.
 * TEST INFRASTRUCTURE ONLY -- called by tests/, the smoke check and the CPU
 * baseline of bench.py; never by the product library, with which it shares no
 * code.
 *
 * What it computes (paweldubiel.com "PagedAttention", "Text order is not a
 * memory address": paging changes where K/V live, not the attention result;
 * mbrenndoerfer.com "Paged Attention > Summary", bullet 3: keys and values are
 * gathered according to the block table):
 *
 *   for sequence s, query head h (KV head g = h / (Hq/Hkv)), tokens t < L_s:
 *     pb  = block_tables[s][t / bs],  off = t % bs
 *     k_t = k_cache[pb][g][off][:],   v_t = v_cache[pb][g][off][:]
 *     x_t = scale * sum_d q[s][h][d] * k_t[d]
 *     out[s][h][:] = sum_t exp(x_t - m) v_t / sum_t exp(x_t - m),  m = max_t x_t
 *
 * Everything is converted from the stored bytes to double and computed in
 * double.  The softmax is the plain two-pass one.  L_s == 0 gives zeros.
 * Layouts: q [B][Hq][D]; caches [NB][Hkv][bs][D]; block_tables [B][max_blocks]
 * int32; seq_lens [B] int32; out [B][Hq][D] double, or [n_sel][D] when a
 * selection of (s, h) pairs is given.
 * Returns 0, or -1 on a bad argument or a table entry outside [0, NB).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { REF_F32 = 0, REF_BF16 = 1, REF_F16 = 2 };

/* IEEE-754 binary32 */
static double dec_f32(const void *base, size_t i) {
    float f;
    memcpy(&f, (const char *)base + 4 * i, 4);
    return (double)f;
}

/* bfloat16: the upper 16 bits of a binary32 */
static double dec_bf16(const void *base, size_t i) {
    uint16_t h;
    uint32_t u;
    float f;
    memcpy(&h, (const char *)base + 2 * i, 2);
    u = (uint32_t)h << 16;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* IEEE-754 binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits */
static double dec_f16(const void *base, size_t i) {
    uint16_t h;
    int e, m;
    double v;
    memcpy(&h, (const char *)base + 2 * i, 2);
    e = (h >> 10) & 31;
    m = h & 1023;
    if (e == 0)
        v = ldexp((double)m, -24);
    else if (e == 31)
        v = m ? NAN : INFINITY;
    else
        v = ldexp((double)(1024 + m), e - 25);
    return (h & 0x8000) ? -v : v;
}

typedef double (*dec_fn)(const void *, size_t);

static dec_fn pick(int dtype) {
    switch (dtype) {
    case REF_F32: return dec_f32;
    case REF_BF16: return dec_bf16;
    case REF_F16: return dec_f16;
    default: return NULL;
    }
}

double attn_ref_decode_value(int dtype, const void *base, long long i) {
    dec_fn f = pick(dtype);
    return f ? f(base, (size_t)i) : NAN;
}

int attn_ref_max_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

static int one_head(double *o, const void *q, const void *kc, const void *vc, dec_fn dec,
                    const int32_t *block_tables, const int32_t *seq_lens, int s, int h,
                    int num_heads, int num_kv_heads, int head_dim, int block_size,
                    int max_blocks, int num_blocks, double scale) {
    const int G = num_heads / num_kv_heads;
    const int g = h / G;
    const int L = seq_lens[s];
    const int D = head_dim;
    double *x, m, den;
    int t, d;

    for (d = 0; d < D; d++) o[d] = 0.0;
    if (L <= 0) return L == 0 ? 0 : -1;
    if ((L + block_size - 1) / block_size > max_blocks) return -1;
    x = (double *)malloc(sizeof(double) * (size_t)L);
    if (!x) return -1;

    /* pass 1: logits, gathered token by token through the block table */
    m = -INFINITY;
    for (t = 0; t < L; t++) {
        int pb = block_tables[(size_t)s * max_blocks + t / block_size];
        int off = t % block_size;
        size_t kbase, qbase = ((size_t)s * num_heads + h) * D;
        double acc = 0.0;
        if (pb < 0 || pb >= num_blocks) { free(x); return -1; }
        kbase = (((size_t)pb * num_kv_heads + g) * block_size + off) * D;
        for (d = 0; d < D; d++) acc += dec(q, qbase + d) * dec(kc, kbase + d);
        x[t] = scale * acc;
        if (x[t] > m) m = x[t];
    }
    /* pass 2: exp-weights, their sum, and the weighted sum of values */
    den = 0.0;
    for (t = 0; t < L; t++) {
        int pb = block_tables[(size_t)s * max_blocks + t / block_size];
        int off = t % block_size;
        size_t vbase = (((size_t)pb * num_kv_heads + g) * block_size + off) * D;
        double w = exp(x[t] - m);
        den += w;
        for (d = 0; d < D; d++) o[d] += w * dec(vc, vbase + d);
    }
    for (d = 0; d < D; d++) o[d] /= den;
    free(x);
    return 0;
}

int attn_ref_decode(double *out, const void *q, const void *k_cache, const void *v_cache,
                    int dtype, const int32_t *block_tables, const int32_t *seq_lens,
                    int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                    int max_blocks, int num_blocks, double scale, const int32_t *sel, int n_sel,
                    int n_threads) {
    dec_fn dec = pick(dtype);
    long long n, i;
    int bad = 0;
    if (!dec || num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        num_heads % num_kv_heads || head_dim <= 0 || block_size <= 0 || max_blocks < 0 ||
        num_blocks <= 0)
        return -1;
    n = sel ? n_sel : (long long)num_seqs * num_heads;
    if (n_threads <= 0) n_threads = attn_ref_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(| : bad)
    for (i = 0; i < n; i++) {
        int s = sel ? sel[2 * i] : (int)(i / num_heads);
        int h = sel ? sel[2 * i + 1] : (int)(i % num_heads);
        if (s < 0 || s >= num_seqs || h < 0 || h >= num_heads) { bad |= 1; continue; }
        bad |= one_head(out + (size_t)i * head_dim, q, k_cache, v_cache, dec, block_tables,
                        seq_lens, s, h, num_heads, num_kv_heads, head_dim, block_size,
                        max_blocks, num_blocks, scale) != 0;
    }
    return bad ? -1 : 0;
}

/*
 * Oracle for multi-token (chunked prefill) attention over the paged cache.
 * The query rows of sequence s are q[cu_q[s] .. cu_q[s+1]): the last
 * n_s = cu_q[s+1] - cu_q[s] positions of the sequence, L_s - n_s .. L_s - 1,
 * whose K/V are already in the cache.  Row r at position p attends, causally,
 * to tokens 0..p, gathered through the block table exactly as in the decode
 * oracle (the decode is the case n_s = 1).
 * Layouts: q [total][Hq][D]; out [total][Hq][D] double.  Returns 0, or -1 on a
 * bad argument (n_s < 0, n_s > L_s, a table entry out of range).
 */
static int prefill_row(double *o, const void *q, size_t qbase, const void *kc, const void *vc,
                       dec_fn dec, const int32_t *table, int L, int g, int num_kv_heads,
                       int head_dim, int block_size, int num_blocks, double scale) {
    const int D = head_dim;
    double *x, m, den;
    int t, d;
    for (d = 0; d < D; d++) o[d] = 0.0;
    x = (double *)malloc(sizeof(double) * (size_t)L);
    if (!x) return -1;
    m = -INFINITY;
    for (t = 0; t < L; t++) {
        int pb = table[t / block_size], off = t % block_size;
        size_t kbase;
        double acc = 0.0;
        if (pb < 0 || pb >= num_blocks) { free(x); return -1; }
        kbase = (((size_t)pb * num_kv_heads + g) * block_size + off) * D;
        for (d = 0; d < D; d++) acc += dec(q, qbase + d) * dec(kc, kbase + d);
        x[t] = scale * acc;
        if (x[t] > m) m = x[t];
    }
    den = 0.0;
    for (t = 0; t < L; t++) {
        int pb = table[t / block_size], off = t % block_size;
        size_t vbase = (((size_t)pb * num_kv_heads + g) * block_size + off) * D;
        double w = exp(x[t] - m);
        den += w;
        for (d = 0; d < D; d++) o[d] += w * dec(vc, vbase + d);
    }
    for (d = 0; d < D; d++) o[d] /= den;
    free(x);
    return 0;
}

int attn_ref_prefill(double *out, const void *q, const void *k_cache, const void *v_cache,
                     int dtype, const int32_t *block_tables, const int32_t *seq_lens,
                     const int32_t *cu_q, int num_seqs, int num_heads, int num_kv_heads,
                     int head_dim, int block_size, int max_blocks, int num_blocks, double scale,
                     int n_threads) {
    dec_fn dec = pick(dtype);
    long long total, i;
    int bad = 0;
    if (!dec || num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        num_heads % num_kv_heads || head_dim <= 0 || block_size <= 0 || max_blocks < 0 ||
        num_blocks <= 0)
        return -1;
    total = num_seqs > 0 ? cu_q[num_seqs] : 0;
    if (n_threads <= 0) n_threads = attn_ref_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(| : bad)
    for (i = 0; i < total * num_heads; i++) {
        const long long r = i / num_heads;
        const int h = (int)(i % num_heads);
        int s = 0, n, L, p;
        while (s + 1 < num_seqs && cu_q[s + 1] <= r) s++;
        n = cu_q[s + 1] - cu_q[s];
        L = seq_lens[s];
        p = L - n + (int)(r - cu_q[s]);
        if (n < 0 || n > L || (L + block_size - 1) / block_size > max_blocks) { bad |= 1; continue; }
        bad |= prefill_row(out + (size_t)i * head_dim, q, ((size_t)r * num_heads + h) * head_dim,
                           k_cache, v_cache, dec, block_tables + (size_t)s * max_blocks, p + 1,
                           h / (num_heads / num_kv_heads), num_kv_heads, head_dim, block_size,
                           num_blocks, scale) != 0;
    }
    return bad ? -1 : 0;
}

/* The same rows as attn_ref_prefill, only the (row, head) pairs listed in
 * sel[2 * j], sel[2 * j + 1]; out[j][D] for pair j. */
int attn_ref_prefill_sel(double *out, const void *q, const void *k_cache, const void *v_cache,
                         int dtype, const int32_t *block_tables, const int32_t *seq_lens,
                         const int32_t *cu_q, int num_seqs, int num_heads, int num_kv_heads,
                         int head_dim, int block_size, int max_blocks, int num_blocks,
                         double scale, const int32_t *sel, int n_sel, int n_threads) {
    dec_fn dec = pick(dtype);
    long long total;
    int j, bad = 0;
    if (!dec || num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 ||
        num_heads % num_kv_heads || head_dim <= 0 || block_size <= 0 || max_blocks < 0 ||
        num_blocks <= 0 || n_sel < 0)
        return -1;
    total = num_seqs > 0 ? cu_q[num_seqs] : 0;
    if (n_threads <= 0) n_threads = attn_ref_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(n_threads) reduction(| : bad)
    for (j = 0; j < n_sel; j++) {
        const long long r = sel[2 * j];
        const int h = sel[2 * j + 1];
        int s = 0, n, L, p;
        if (r < 0 || r >= total || h < 0 || h >= num_heads) { bad |= 1; continue; }
        while (s + 1 < num_seqs && cu_q[s + 1] <= r) s++;
        n = cu_q[s + 1] - cu_q[s];
        L = seq_lens[s];
        p = L - n + (int)(r - cu_q[s]);
        if (n < 0 || n > L || (L + block_size - 1) / block_size > max_blocks) { bad |= 1; continue; }
        bad |= prefill_row(out + (size_t)j * head_dim, q, ((size_t)r * num_heads + h) * head_dim,
                           k_cache, v_cache, dec, block_tables + (size_t)s * max_blocks, p + 1,
                           h / (num_heads / num_kv_heads), num_kv_heads, head_dim, block_size,
                           num_blocks, scale) != 0;
    }
    return bad ? -1 : 0;
}

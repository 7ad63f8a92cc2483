/*
 * duo_oracle.c -- float64 CPU oracle for DuoAttention hybrid-GQA attention.
 *
 * TEST INFRASTRUCTURE.  This file is the slow, plain statement of what the
 * attention path computes.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load it.  It shares no code, header,
 * table or helper with the CUDA library; it reads inputs as raw bf16 bit
 * patterns and computes every sum in double precision, one output row at a
 * time, in the order the definition states.
 *
 * Sources (web pages on the subject):
 *  - "DuoAttention Laguna Adapter" model card, sections Summary and Why It
 *    Works: every KV head is either a full-context head, which keeps all
 *    prior tokens, or a streaming head, which keeps only a sink window
 *    (64 tokens) plus a recent window (256 tokens).
 *  - "Laguna attention: sliding window and RoPE" (Laguna-M.1-8bit article),
 *    section on sliding-window attention: each token attends only to a fixed
 *    window of preceding tokens, chosen per layer through layer_types.
 *  - "Laguna XS 2.1 sliding-window attention" article, section 3 (attention
 *    sink optimisation): sliding-window layers carry an optional learnable
 *    sink term.  Read here as one float logit per query head that joins the
 *    softmax denominator with a zero value vector, added unscaled.
 *  - Laguna-XS-2.1 SGLang cookbook, section 1: 48 query heads, 8 KV heads,
 *    window 512.  Query head h reads KV head floor(h / (Hq / Hkv)).
 *
 * Readings where the pages are silent: the recent window includes the
 * query itself (a query at position i keeps keys j with j > i - recent);
 * the sink and recent windows may overlap and their union is attended; the
 * exported log-sum-exp includes the sink term; a sliding layer's cache is a
 * ring of `window` slots per KV head (the streaming layout with no sink).
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC -o liboracle.so duo_oracle.c -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Problem description as the oracle sees it. */
typedef struct {
    int32_t batch;
    int32_t num_q_heads;
    int32_t num_kv_heads;
    int32_t head_dim;
    int32_t sink;          /* streaming heads: tokens kept from the start  */
    int32_t recent;        /* streaming heads: most recent tokens kept     */
    int32_t window;        /* > 0: sliding-window layer; 0: DuoAttention   */
    double softmax_scale;  /* multiplies q.k; the sink logit is not scaled */
    const uint8_t *full_mask;  /* [num_kv_heads], 1 = full-context head    */
    const float *sink_logit;   /* [num_q_heads] or NULL                     */
} oracle_params;

/* A KV cache held in host memory, laid out head-major like the device one:
 *   full_k/full_v: [batch][n_full][capacity][head_dim]
 *   strm_k/strm_v: [batch][n_strm][sink + recent][head_dim]   (Duo layer)
 *                  [batch][num_kv_heads][window][head_dim]     (sliding)
 * seq_len[b] counts the tokens appended so far; ring_head[b] is the ring
 * slot (0 .. ring size - 1) that the next ring write goes to. */
typedef struct {
    uint16_t *full_k, *full_v;
    int64_t capacity;
    uint16_t *strm_k, *strm_v;
    int32_t *seq_len, *ring_head;
} oracle_cache;

enum { KIND_FULL = 0, KIND_STREAMING = 1, KIND_SLIDING = 2 };

static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;  /* bf16 is the top half of a float */
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

int oracle_head_kind(const oracle_params *p, int32_t kv_head) {
    if (p->window > 0) return KIND_SLIDING;
    return p->full_mask[kv_head] ? KIND_FULL : KIND_STREAMING;
}

/* Number of full heads with index below kv_head (its slot in the full cache). */
static int32_t full_rank(const oracle_params *p, int32_t kv_head) {
    int32_t r = 0;
    for (int32_t g = 0; g < kv_head; ++g) r += (oracle_head_kind(p, g) == KIND_FULL);
    return r;
}

/* Number of non-full heads with index below kv_head (slot in the ring cache). */
static int32_t ring_rank(const oracle_params *p, int32_t kv_head) {
    int32_t r = 0;
    for (int32_t g = 0; g < kv_head; ++g) r += (oracle_head_kind(p, g) != KIND_FULL);
    return r;
}

static int32_t count_full(const oracle_params *p) { return full_rank(p, p->num_kv_heads); }

/* Sink and recent sizes of the ring cache for this layer. */
static int32_t ring_sink(const oracle_params *p) { return p->window > 0 ? 0 : p->sink; }
static int32_t ring_recent(const oracle_params *p) { return p->window > 0 ? p->window : p->recent; }

/* The attended set: does the query at position i read the key at position j?
 *  full:      0 <= j <= i
 *  streaming: j <= i and (j < sink or j > i - recent)
 *  sliding:   j <= i and j > i - window                                     */
int oracle_attended(const oracle_params *p, int32_t kv_head, int64_t i, int64_t j) {
    if (j < 0 || j > i) return 0;
    switch (oracle_head_kind(p, kv_head)) {
    case KIND_FULL: return 1;
    case KIND_STREAMING: return j < p->sink || j > i - p->recent;
    default: return j > i - p->window;
    }
}

/* Counts attended (i, j) pairs for 0 <= i < L, one KV head. */
int64_t oracle_count_pairs(const oracle_params *p, int32_t kv_head, int64_t L) {
    int64_t total = 0;
#pragma omp parallel for reduction(+ : total) schedule(dynamic, 64)
    for (int64_t i = 0; i < L; ++i)
        for (int64_t j = 0; j <= i; ++j) total += oracle_attended(p, kv_head, i, j);
    return total;
}

/* softmax over one row of scores s[0..n) (already scaled), plus the sink
 * logit when present; writes out[d] = sum_j e^{s_j - m} v_j / Z and returns
 * LSE = m + ln Z.  vrow(j) gives the value row of the j-th listed key. */
static double softmax_row(int n, const double *s, const uint16_t *const *vrows, int D,
                          int has_sink, double sigma, double *out) {
    if (n == 0 && !has_sink) {  /* nothing attended: zero output, LSE = -inf */
        for (int d = 0; d < D; ++d) out[d] = 0.0;
        return -INFINITY;
    }
    double m = -INFINITY;
    for (int j = 0; j < n; ++j) m = fmax(m, s[j]);
    if (has_sink) m = fmax(m, sigma);
    double Z = 0.0;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int j = 0; j < n; ++j) {
        double w = exp(s[j] - m);
        Z += w;
        for (int d = 0; d < D; ++d) out[d] += w * bf16_value(vrows[j][d]);
    }
    if (has_sink) Z += exp(sigma - m);
    for (int d = 0; d < D; ++d) out[d] /= Z;
    return m + log(Z);
}

static double dot_bf16(const uint16_t *a, const uint16_t *b, int D) {
    double acc = 0.0;
    for (int d = 0; d < D; ++d) acc += bf16_value(a[d]) * bf16_value(b[d]);
    return acc;
}

/* Prefill attention over an empty cache.
 *   q: [B][L][Hq][D], k, v: [B][L][Hkv][D], bf16 bits.
 *   rows: flat row ids r = (b*Hq + h)*L + i, or NULL for every row.
 *   out: [n_rows][D] float64, lse: [n_rows] float64.
 * Each row: the attended keys of query i under its KV head's rule. */
int oracle_attn_prefill(const oracle_params *p, const uint16_t *q, const uint16_t *k,
                        const uint16_t *v, int64_t L, const int64_t *rows, int64_t n_rows,
                        double *out, double *lse) {
    const int Hq = p->num_q_heads, Hkv = p->num_kv_heads, D = p->head_dim;
    if (Hq % Hkv) return -1;
    const int group = Hq / Hkv;
    const int64_t total = (int64_t)p->batch * Hq * L;
    if (!rows) n_rows = total;
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)(L > 0 ? L : 1));
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)(L > 0 ? L : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t t = 0; t < n_rows; ++t) {
            const int64_t r = rows ? rows[t] : t;
            if (r < 0 || r >= total) { bad = 1; continue; }
            const int64_t i = r % L;
            const int h = (int)((r / L) % Hq);
            const int64_t b = r / L / Hq;
            const int g = h / group;
            const uint16_t *qi = q + ((b * L + i) * Hq + h) * D;
            int n = 0;
            for (int64_t j = 0; j <= i; ++j) {
                if (!oracle_attended(p, g, i, j)) continue;
                const uint16_t *kj = k + ((b * L + j) * Hkv + g) * D;
                s[n] = p->softmax_scale * dot_bf16(qi, kj, D);
                vr[n] = v + ((b * L + j) * Hkv + g) * D;
                ++n;
            }
            const int has_sink = p->sink_logit != NULL;
            const double sigma = has_sink ? (double)p->sink_logit[h] : 0.0;
            lse[t] = softmax_row(n, s, vr, D, has_sink, sigma, out + t * D);
        }
        free(s);
        free((void *)vr);
    }
    return bad ? -2 : 0;
}

/* Appends n_new tokens per sequence, one token at a time:
 * position p = seq_len; a full head stores the token at row p of its
 * full-cache slot; another head stores it at ring slot p if p < sink, else
 * at slot sink + ring_head, and ring_head then moves to the next slot
 * (mod recent).  k, v: [B][n_new][Hkv][D] bf16 bits. */
int oracle_kv_append(const oracle_params *p, oracle_cache *c, const uint16_t *k,
                     const uint16_t *v, int32_t n_new) {
    const int Hkv = p->num_kv_heads, D = p->head_dim;
    const int32_t n_full = count_full(p), n_ring = Hkv - n_full;
    const int32_t S = ring_sink(p), R = ring_recent(p), slots = S + R;
    for (int32_t b = 0; b < p->batch; ++b) {
        for (int32_t t = 0; t < n_new; ++t) {
            const int64_t pos = c->seq_len[b];
            if (n_full > 0 && pos >= c->capacity) return -1;
            for (int32_t g = 0; g < Hkv; ++g) {
                const uint16_t *ks = k + (((int64_t)b * n_new + t) * Hkv + g) * D;
                const uint16_t *vs = v + (((int64_t)b * n_new + t) * Hkv + g) * D;
                uint16_t *kd, *vd;
                if (oracle_head_kind(p, g) == KIND_FULL) {
                    const int64_t row = (((int64_t)b * n_full + full_rank(p, g)) * c->capacity + pos);
                    kd = c->full_k + row * D;
                    vd = c->full_v + row * D;
                } else {
                    const int64_t slot = pos < S ? pos : S + c->ring_head[b];
                    const int64_t row = ((int64_t)b * n_ring + ring_rank(p, g)) * slots + slot;
                    kd = c->strm_k + row * D;
                    vd = c->strm_v + row * D;
                }
                memcpy(kd, ks, sizeof(uint16_t) * (size_t)D);
                memcpy(vd, vs, sizeof(uint16_t) * (size_t)D);
            }
            if (pos >= S) c->ring_head[b] = (c->ring_head[b] + 1) % R;
            c->seq_len[b] = (int32_t)(pos + 1);
        }
    }
    return 0;
}

/* One-token decode against the cache.  The query sits at position n - 1,
 * n = seq_len[b].  q: [B][Hq][D] bf16 bits.  rows: flat ids b*Hq + h, or
 * NULL for all.  A full head reads cache rows 0..n-1.  A ring head reads
 * the sink slots 0..min(n, sink)-1 and the c = min(max(n - sink, 0), recent)
 * ring slots written last, i.e. the c slots before ring_head, cyclically. */
int oracle_attn_decode(const oracle_params *p, const oracle_cache *c, const uint16_t *q,
                       const int64_t *rows, int64_t n_rows, double *out, double *lse) {
    const int Hq = p->num_q_heads, Hkv = p->num_kv_heads, D = p->head_dim;
    if (Hq % Hkv) return -1;
    const int group = Hq / Hkv;
    const int32_t n_full = count_full(p), n_ring = Hkv - n_full;
    const int32_t S = ring_sink(p), R = ring_recent(p), slots = S + R;
    const int64_t total = (int64_t)p->batch * Hq;
    if (!rows) n_rows = total;
    int64_t max_n = 1;
    for (int32_t b = 0; b < p->batch; ++b)
        if (c->seq_len[b] > max_n) max_n = c->seq_len[b];
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)max_n);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)max_n);
#pragma omp for schedule(dynamic, 1)
        for (int64_t t = 0; t < n_rows; ++t) {
            const int64_t r = rows ? rows[t] : t;
            if (r < 0 || r >= total) { bad = 1; continue; }
            const int64_t b = r / Hq;
            const int h = (int)(r % Hq);
            const int g = h / group;
            const int64_t n = c->seq_len[b];
            const uint16_t *qh = q + (b * Hq + h) * D;
            int m = 0;
            if (oracle_head_kind(p, g) == KIND_FULL) {
                const int64_t base = ((b * n_full + full_rank(p, g)) * c->capacity) * D;
                for (int64_t j = 0; j < n; ++j) {
                    s[m] = p->softmax_scale * dot_bf16(qh, c->full_k + base + j * D, D);
                    vr[m++] = c->full_v + base + j * D;
                }
            } else {
                const int64_t base = ((b * n_ring + ring_rank(p, g)) * slots) * D;
                const int64_t n_sink = n < S ? n : S;
                int64_t cnt = n - S;
                if (cnt < 0) cnt = 0;
                if (cnt > R) cnt = R;
                for (int64_t j = 0; j < n_sink; ++j) {
                    s[m] = p->softmax_scale * dot_bf16(qh, c->strm_k + base + j * D, D);
                    vr[m++] = c->strm_v + base + j * D;
                }
                for (int64_t e = 0; e < cnt; ++e) {
                    const int64_t slot = S + (((int64_t)c->ring_head[b] - cnt + e) % R + R) % R;
                    s[m] = p->softmax_scale * dot_bf16(qh, c->strm_k + base + slot * D, D);
                    vr[m++] = c->strm_v + base + slot * D;
                }
            }
            const int has_sink = p->sink_logit != NULL;
            const double sigma = has_sink ? (double)p->sink_logit[h] : 0.0;
            lse[t] = softmax_row(m, s, vr, D, has_sink, sigma, out + t * D);
        }
        free(s);
        free((void *)vr);
    }
    return bad ? -2 : 0;
}

/* Block decode: a block of qlen query tokens (a verify block) against the
 * cache as it stands BEFORE the block is appended.  Query t of sequence b sits
 * at position i = n + t, n = seq_len[b], and attends to the keys its head's
 * rule allows at i: the cached ones (a full head: rows 0..n-1; a ring head:
 * its sink slots, and the ring slots holding a position j > i - recent, where
 * the ring slot written d-th to last holds position n - 1 - d) and the block's
 * own keys u <= t (positions n..i) that the same rule allows, given in kb, vb
 * [B][qlen][Hkv][D].
 * q: [B][qlen][Hq][D].  rows: flat ids (b*qlen + t)*Hq + h, or NULL for all. */
int oracle_attn_decode_block(const oracle_params *p, const oracle_cache *c, const uint16_t *q,
                             const uint16_t *kb, const uint16_t *vb, int32_t qlen,
                             const int64_t *rows, int64_t n_rows, double *out, double *lse) {
    const int Hq = p->num_q_heads, Hkv = p->num_kv_heads, D = p->head_dim;
    if (Hq % Hkv || qlen < 1) return -1;
    const int group = Hq / Hkv;
    const int32_t n_full = count_full(p), n_ring = Hkv - n_full;
    const int32_t S = ring_sink(p), R = ring_recent(p), slots = S + R;
    const int64_t total = (int64_t)p->batch * qlen * Hq;
    if (!rows) n_rows = total;
    int64_t max_keys = 1;
    for (int32_t b = 0; b < p->batch; ++b)
        if (c->seq_len[b] + qlen > max_keys) max_keys = c->seq_len[b] + qlen;
    int bad = 0;
#pragma omp parallel
    {
        double *s = (double *)malloc(sizeof(double) * (size_t)max_keys);
        const uint16_t **vr = (const uint16_t **)malloc(sizeof(void *) * (size_t)max_keys);
#pragma omp for schedule(dynamic, 1)
        for (int64_t x = 0; x < n_rows; ++x) {
            const int64_t r = rows ? rows[x] : x;
            if (r < 0 || r >= total) { bad = 1; continue; }
            const int h = (int)(r % Hq);
            const int64_t t = (r / Hq) % qlen;
            const int64_t b = r / Hq / qlen;
            const int g = h / group;
            const int64_t n = c->seq_len[b];
            const int64_t i = n + t;                   /* the query's position */
            const uint16_t *qh = q + ((b * qlen + t) * Hq + h) * D;
            int m = 0;
            if (oracle_head_kind(p, g) == KIND_FULL) {
                const int64_t base = ((b * n_full + full_rank(p, g)) * c->capacity) * D;
                for (int64_t j = 0; j < n; ++j) {
                    s[m] = p->softmax_scale * dot_bf16(qh, c->full_k + base + j * D, D);
                    vr[m++] = c->full_v + base + j * D;
                }
            } else {
                const int64_t base = ((b * n_ring + ring_rank(p, g)) * slots) * D;
                const int64_t n_sink = n < S ? n : S;
                int64_t cnt = n - S;
                if (cnt < 0) cnt = 0;
                if (cnt > R) cnt = R;
                for (int64_t j = 0; j < n_sink; ++j) {
                    s[m] = p->softmax_scale * dot_bf16(qh, c->strm_k + base + j * D, D);
                    vr[m++] = c->strm_v + base + j * D;
                }
                for (int64_t d = 0; d < cnt; ++d) {    /* d-th to last written: position n-1-d */
                    const int64_t pos = n - 1 - d;
                    if (pos <= i - R) continue;        /* outside the query's recent window */
                    const int64_t slot = S + (((int64_t)c->ring_head[b] - 1 - d) % R + R) % R;
                    s[m] = p->softmax_scale * dot_bf16(qh, c->strm_k + base + slot * D, D);
                    vr[m++] = c->strm_v + base + slot * D;
                }
            }
            for (int64_t u = 0; u <= t; ++u) {         /* the block's keys up to the query */
                const int64_t j = n + u;
                if (oracle_head_kind(p, g) != KIND_FULL && !(j < S || j > i - R)) continue;
                const int64_t kr = ((b * qlen + u) * Hkv + g) * D;
                s[m] = p->softmax_scale * dot_bf16(qh, kb + kr, D);
                vr[m++] = vb + kr;
            }
            const int has_sink = p->sink_logit != NULL;
            const double sigma = has_sink ? (double)p->sink_logit[h] : 0.0;
            lse[x] = softmax_row(m, s, vr, D, has_sink, sigma, out + x * D);
        }
        free(s);
        free((void *)vr);
    }
    return bad ? -2 : 0;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}

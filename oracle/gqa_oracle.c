/*
 * Plain fp64 CPU oracle for grouped-query attention.  TEST INFRASTRUCTURE ONLY:
 * only the tests, the smoke check and the bench's CPU-baseline leg may load it.
 * It shares no code, header or constant with the CUDA library.
 *
 * What it computes (the plain definition, written out):
 *   "Evolution of AI Attention Mechanisms" (toolsku), section "MHA Mathematical
 *   Formulation": per head, Attn = softmax(Q K^T * scale) V, heads being
 *   contiguous d_h slices of the hidden dimension;
 *   same page, "GQA Implementation": with n_rep = h / n_kv, K/V head g is
 *   repeated n_rep times (expand then reshape), so query head i reads KV
 *   head i / n_rep;
 *   same page, "MHA Implementation": masked scores are set to -inf before the
 *   softmax, and past K/V are concatenated in front of the new ones (so new
 *   queries are the LAST S_q positions: bottom-right causal alignment);
 *   "Attention variants" (saadho), "What this topic covers": FlashAttention
 *   computes this same exact result, so the oracle is the untiled definition.
 *
 * For every (batch b, query head i) the full score matrix of the requested
 * query rows against all keys is materialised in fp64, masked, soft-maxed row
 * by row (max subtracted, as a softmax is usually evaluated), and multiplied
 * by V.  Inputs are bf16 bit patterns; each is widened exactly to fp64.
 *
 * Decode caches may also be stored as 8-bit floats or in pages:
 *   "Multi-Query Attention (MQA)" (inferensys glossary), paragraph "KV cache
 *   quantization": K and V are kept in a lower precision (FP8 among the
 *   formats named) with scaling factors; "Multi-query attention"
 *   (pranaymahendrakar), "Interaction with other techniques": an fp8 cache
 *   halves the bytes per element.  Reading taken here: the OCP E4M3 format
 *   (no infinities) with one fp32 scale per KV head for K and one for V; a
 *   cached value is code_value * scale, widened exactly to fp64 (4 + 24
 *   significant bits fit in 53).
 *   Same glossary, paragraph "PagedAttention": each sequence's cache is cut
 *   into fixed-size pages that may lie anywhere in memory.  Reading taken
 *   here: token t of sequence b is slot t % page_size of page
 *   block_table[b][t / page_size], a page holding [page_size, n_kv, d].
 * Either way the cached rows are first gathered into plain fp64 K and V
 * matrices, then the same untiled attention runs.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

static double bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * OCP 8-bit floating point E4M3 (the variant without infinities): sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits.  Exponent field 0 encodes the
 * subnormals (m / 8) * 2^-6; exponent 15 with mantissa 7 is NaN; every other
 * code is (1 + m / 8) * 2^(e - 7), so the largest finite magnitude is 448.
 */
double oracle_e4m3_value(uint8_t code) {
    int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) mag = ldexp((double)m / 8.0, -6);
    else mag = ldexp(1.0 + (double)m / 8.0, e - 7);
    return sign ? -mag : mag;
}

/*
 * One attention unit on fp64 operands.  q_rows: nr query vectors of length d.
 * kd/vd: nk x d keys and values.  visible[r]: query row r sees keys
 * j < visible[r].  out: nr x d.  probs (optional): nr x nk softmax matrix.
 */
static int attend_f64(const double *q_rows, int nr, const double *kd, const double *vd, int nk, int d,
                      const int *visible, double scale, double *out, double *probs) {
    double *S = (double *)malloc(sizeof(double) * (size_t)(nr > 0 ? nr : 1) * (size_t)(nk > 0 ? nk : 1));
    if (!S) return -1;
    /* scores, with the mask */
    for (int r = 0; r < nr; ++r)
        for (int j = 0; j < nk; ++j) {
            double *s = &S[(size_t)r * nk + j];
            if (j >= visible[r]) { *s = -INFINITY; continue; }
            double acc = 0.0;
            for (int c = 0; c < d; ++c) acc += q_rows[(size_t)r * d + c] * kd[(size_t)j * d + c];
            *s = acc * scale;
        }
    /* row softmax, then P V */
    for (int r = 0; r < nr; ++r) {
        double *srow = &S[(size_t)r * nk];
        double *orow = &out[(size_t)r * d];
        for (int c = 0; c < d; ++c) orow[c] = 0.0;
        if (visible[r] <= 0) {            /* no key: the row is defined as zero */
            if (probs) for (int j = 0; j < nk; ++j) probs[(size_t)r * nk + j] = 0.0;
            continue;
        }
        double m = -INFINITY;
        for (int j = 0; j < nk; ++j) if (srow[j] > m) m = srow[j];
        double sum = 0.0;
        for (int j = 0; j < nk; ++j) {
            srow[j] = (srow[j] == -INFINITY) ? 0.0 : exp(srow[j] - m);
            sum += srow[j];
        }
        for (int j = 0; j < nk; ++j) srow[j] /= sum;
        if (probs) memcpy(&probs[(size_t)r * nk], srow, sizeof(double) * (size_t)nk);
        for (int j = 0; j < nk; ++j) {
            double p = srow[j];
            if (p == 0.0) continue;
            for (int c = 0; c < d; ++c) orow[c] += p * vd[(size_t)j * d + c];
        }
    }
    free(S);
    return 0;
}

/* The same unit with bf16 K/V rows read through a row stride (in elements). */
static int attend(const double *q_rows, int nr, const uint16_t *k0, const uint16_t *v0,
                  long kv_row_stride, int nk, int d, const int *visible, double scale,
                  double *out, double *probs) {
    double *kd = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * (size_t)d);
    double *vd = (double *)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1) * (size_t)d);
    if (!kd || !vd) { free(kd); free(vd); return -1; }
    for (int j = 0; j < nk; ++j)
        for (int c = 0; c < d; ++c) {
            kd[(size_t)j * d + c] = bf16_value(k0[(size_t)j * kv_row_stride + c]);
            vd[(size_t)j * d + c] = bf16_value(v0[(size_t)j * kv_row_stride + c]);
        }
    int rc = attend_f64(q_rows, nr, kd, vd, nk, d, visible, scale, out, probs);
    free(kd); free(vd);
    return rc;
}

/* ------------------------------------------------------------------------ */
/* thread pool over units                                                    */

typedef struct {
    int kind;                 /* 0 prefill, 1 decode */
    const uint16_t *q, *k, *v;
    const int32_t *seqlens;
    const long *offsets;      /* decode: first cache row of each sequence */
    /* general decode (kind 2): cache element format and page table */
    const void *kc, *vc;      /* caches: bf16 bits (fmt 0) or E4M3 codes (fmt 1) */
    int fmt;
    const float *k_scale, *v_scale;   /* fmt 1: one scale per KV head */
    const int32_t *block_table;       /* NULL: packed layout */
    int max_blocks, page_size;
    double *out;
    int B, S_q, S_kv, h, n_kv, d, causal;
    double scale;
    /* sampled prefill rows: triplets (b, i, r); NULL = every row */
    const int32_t *sample;
    int n_sample;
    int n_units;
    int n_threads;
    int failed;
} job_t;

typedef struct { job_t *job; int tid; } worker_arg_t;

static void run_prefill_unit(job_t *J, int b, int i, const int *rows, int nr, double *out_rows) {
    int G = J->h / J->n_kv;
    int g = i / G;                                  /* the group of query head i */
    int d = J->d;
    double *qd = (double *)malloc(sizeof(double) * (size_t)nr * d);
    int *vis = (int *)malloc(sizeof(int) * (size_t)nr);
    if (!qd || !vis) { free(qd); free(vis); J->failed = 1; return; }
    for (int t = 0; t < nr; ++t) {
        int r = rows[t];
        const uint16_t *qrow = J->q + (((size_t)b * J->S_q + r) * J->h + i) * d;
        for (int c = 0; c < d; ++c) qd[(size_t)t * d + c] = bf16_value(qrow[c]);
        int lim = J->S_kv;
        if (J->causal) {
            int last = r + (J->S_kv - J->S_q);   /* bottom-right alignment */
            if (last + 1 < lim) lim = last + 1;
            if (lim < 0) lim = 0;
        }
        vis[t] = lim;
    }
    const uint16_t *k0 = J->k + ((size_t)b * J->S_kv * J->n_kv + g) * d;
    const uint16_t *v0 = J->v + ((size_t)b * J->S_kv * J->n_kv + g) * d;
    if (attend(qd, nr, k0, v0, (long)J->n_kv * d, J->S_kv, d, vis, J->scale, out_rows, NULL))
        J->failed = 1;
    free(qd); free(vis);
}

static void run_decode_unit(job_t *J, int b, int i) {
    int G = J->h / J->n_kv;
    int g = i / G;
    int d = J->d;
    int L = J->seqlens[b];
    double *orow = J->out + ((size_t)b * J->h + i) * d;
    if (L <= 0) { for (int c = 0; c < d; ++c) orow[c] = 0.0; return; }
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    if (!qd) { J->failed = 1; return; }
    const uint16_t *qrow = J->q + ((size_t)b * J->h + i) * d;
    for (int c = 0; c < d; ++c) qd[c] = bf16_value(qrow[c]);
    const uint16_t *k0 = J->k + ((size_t)J->offsets[b] * J->n_kv + g) * d;
    const uint16_t *v0 = J->v + ((size_t)J->offsets[b] * J->n_kv + g) * d;
    int vis = L;
    if (attend(qd, 1, k0, v0, (long)J->n_kv * d, L, d, &vis, J->scale, orow, NULL)) J->failed = 1;
    free(qd);
}

/* Cache row of token t of sequence b (in units of n_kv * d elements). */
static long cache_row(const job_t *J, int b, int t) {
    if (!J->block_table) return J->offsets[b] + t;
    int page = J->block_table[(size_t)b * J->max_blocks + t / J->page_size];
    return (long)page * J->page_size + t % J->page_size;
}

static double cache_value(const job_t *J, const void *cache, const float *sc, long idx, int g) {
    if (J->fmt == 0) return bf16_value(((const uint16_t *)cache)[idx]);
    return oracle_e4m3_value(((const uint8_t *)cache)[idx]) * (double)sc[g];
}

static void run_decode_general_unit(job_t *J, int b, int i) {
    int G = J->h / J->n_kv;
    int g = i / G;
    int d = J->d;
    int L = J->seqlens[b];
    double *orow = J->out + ((size_t)b * J->h + i) * d;
    if (L <= 0) { for (int c = 0; c < d; ++c) orow[c] = 0.0; return; }
    double *qd = (double *)malloc(sizeof(double) * (size_t)d);
    double *kd = (double *)malloc(sizeof(double) * (size_t)L * d);
    double *vd = (double *)malloc(sizeof(double) * (size_t)L * d);
    if (!qd || !kd || !vd) { free(qd); free(kd); free(vd); J->failed = 1; return; }
    const uint16_t *qrow = J->q + ((size_t)b * J->h + i) * d;
    for (int c = 0; c < d; ++c) qd[c] = bf16_value(qrow[c]);
    /* gather the cached rows of KV head g */
    for (int t = 0; t < L; ++t) {
        long base = (cache_row(J, b, t) * J->n_kv + g) * (long)d;
        for (int c = 0; c < d; ++c) {
            kd[(size_t)t * d + c] = cache_value(J, J->kc, J->k_scale, base + c, g);
            vd[(size_t)t * d + c] = cache_value(J, J->vc, J->v_scale, base + c, g);
        }
    }
    if (attend_f64(qd, 1, kd, vd, L, d, &L, J->scale, orow, NULL)) J->failed = 1;
    free(qd); free(kd); free(vd);
}

static void *worker(void *p) {
    worker_arg_t *a = (worker_arg_t *)p;
    job_t *J = a->job;
    for (int u = a->tid; u < J->n_units; u += J->n_threads) {
        if (J->kind == 1) {
            run_decode_unit(J, u / J->h, u % J->h);
        } else if (J->kind == 2) {
            run_decode_general_unit(J, u / J->h, u % J->h);
        } else if (J->sample) {
            const int32_t *s = J->sample + 3 * (size_t)u;
            int r = s[2];
            run_prefill_unit(J, s[0], s[1], &r, 1, J->out + (size_t)u * J->d);
        } else {
            int b = u / J->h, i = u % J->h;
            int *rows = (int *)malloc(sizeof(int) * (size_t)J->S_q);
            double *tmp = (double *)malloc(sizeof(double) * (size_t)J->S_q * J->d);
            if (!rows || !tmp) { free(rows); free(tmp); J->failed = 1; continue; }
            for (int r = 0; r < J->S_q; ++r) rows[r] = r;
            run_prefill_unit(J, b, i, rows, J->S_q, tmp);
            /* scatter to out[b, r, i, :] */
            for (int r = 0; r < J->S_q; ++r)
                memcpy(J->out + (((size_t)b * J->S_q + r) * J->h + i) * J->d,
                       tmp + (size_t)r * J->d, sizeof(double) * (size_t)J->d);
            free(rows); free(tmp);
        }
    }
    return NULL;
}

static int run_job(job_t *J, int n_threads) {
    if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (n_threads < 1) n_threads = 1;
    if (n_threads > J->n_units) n_threads = J->n_units > 0 ? J->n_units : 1;
    J->n_threads = n_threads;
    J->failed = 0;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)n_threads);
    worker_arg_t *args = (worker_arg_t *)malloc(sizeof(worker_arg_t) * (size_t)n_threads);
    if (!th || !args) { free(th); free(args); return -1; }
    for (int t = 0; t < n_threads; ++t) {
        args[t].job = J; args[t].tid = t;
        pthread_create(&th[t], NULL, worker, &args[t]);
    }
    for (int t = 0; t < n_threads; ++t) pthread_join(th[t], NULL);
    free(th); free(args);
    return J->failed ? -1 : 0;
}

static int check_shape(int B, int h, int n_kv, int d) {
    return B > 0 && h > 0 && n_kv > 0 && d > 0 && h % n_kv == 0;
}

/* ------------------------------------------------------------------------ */
/* exported entry points                                                     */

/* Causal or full prefill.  q [B,S_q,h,d], k/v [B,S_kv,n_kv,d] bf16 bits,
 * out [B,S_q,h,d] fp64.  Returns 0, or -1 on bad arguments / no memory. */
int oracle_prefill(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *out,
                   int B, int S_q, int S_kv, int h, int n_kv, int d, int causal,
                   double scale, int n_threads) {
    if (!check_shape(B, h, n_kv, d) || S_q <= 0 || S_kv <= 0) return -1;
    job_t J = {0};
    J.kind = 0; J.q = q; J.k = k; J.v = v; J.out = out;
    J.B = B; J.S_q = S_q; J.S_kv = S_kv; J.h = h; J.n_kv = n_kv; J.d = d;
    J.causal = causal; J.scale = scale;
    J.n_units = B * h;
    return run_job(&J, n_threads);
}

/* The same, for selected query rows only: sample holds n triplets (b, i, r);
 * out is n x d, row t being output row r of query head i in batch b. */
int oracle_prefill_rows(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *out,
                        int B, int S_q, int S_kv, int h, int n_kv, int d, int causal,
                        double scale, const int32_t *sample, int n, int n_threads) {
    if (!check_shape(B, h, n_kv, d) || S_q <= 0 || S_kv <= 0 || n < 0) return -1;
    for (int t = 0; t < n; ++t) {
        const int32_t *s = sample + 3 * (size_t)t;
        if (s[0] < 0 || s[0] >= B || s[1] < 0 || s[1] >= h || s[2] < 0 || s[2] >= S_q) return -1;
    }
    job_t J = {0};
    J.kind = 0; J.q = q; J.k = k; J.v = v; J.out = out;
    J.B = B; J.S_q = S_q; J.S_kv = S_kv; J.h = h; J.n_kv = n_kv; J.d = d;
    J.causal = causal; J.scale = scale; J.sample = sample; J.n_sample = n;
    J.n_units = n;
    return run_job(&J, n_threads);
}

/* One decode step.  q [B,h,d]; caches packed [sum(max(seqlens,0)), n_kv, d]
 * (sequence b starting at row sum of the earlier lengths); out [B,h,d] fp64.
 * Query head i of sequence b attends to all seqlens[b] cached tokens of KV
 * head i / (h / n_kv); a length <= 0 gives a zero row. */
int oracle_decode(const uint16_t *q, const uint16_t *k_cache, const uint16_t *v_cache,
                  const int32_t *seqlens, double *out, int B, int h, int n_kv, int d,
                  double scale, int n_threads) {
    if (!check_shape(B, h, n_kv, d)) return -1;
    long *off = (long *)malloc(sizeof(long) * (size_t)B);
    if (!off) return -1;
    long acc = 0;
    for (int b = 0; b < B; ++b) { off[b] = acc; if (seqlens[b] > 0) acc += seqlens[b]; }
    job_t J = {0};
    J.kind = 1; J.q = q; J.k = k_cache; J.v = v_cache; J.seqlens = seqlens; J.offsets = off;
    J.out = out; J.B = B; J.h = h; J.n_kv = n_kv; J.d = d; J.scale = scale;
    J.n_units = B * h;
    int rc = run_job(&J, n_threads);
    free(off);
    return rc;
}

/* The softmax matrix of one prefill unit (b, i): probs is S_q x S_kv. */
int oracle_prefill_probs(const uint16_t *q, const uint16_t *k, const uint16_t *v, double *probs,
                         int B, int S_q, int S_kv, int h, int n_kv, int d, int causal,
                         double scale, int b, int i) {
    if (!check_shape(B, h, n_kv, d) || S_q <= 0 || S_kv <= 0) return -1;
    if (b < 0 || b >= B || i < 0 || i >= h) return -1;
    int G = h / n_kv, g = i / G;
    double *qd = (double *)malloc(sizeof(double) * (size_t)S_q * d);
    double *o = (double *)malloc(sizeof(double) * (size_t)S_q * d);
    int *vis = (int *)malloc(sizeof(int) * (size_t)S_q);
    if (!qd || !o || !vis) { free(qd); free(o); free(vis); return -1; }
    for (int r = 0; r < S_q; ++r) {
        const uint16_t *qrow = q + (((size_t)b * S_q + r) * h + i) * d;
        for (int c = 0; c < d; ++c) qd[(size_t)r * d + c] = bf16_value(qrow[c]);
        int lim = S_kv;
        if (causal) { int last = r + (S_kv - S_q); if (last + 1 < lim) lim = last + 1; if (lim < 0) lim = 0; }
        vis[r] = lim;
    }
    int rc = attend(qd, S_q, k + ((size_t)b * S_kv * n_kv + g) * d, v + ((size_t)b * S_kv * n_kv + g) * d,
                    (long)n_kv * d, S_kv, d, vis, scale, o, probs);
    free(qd); free(o); free(vis);
    return rc;
}

/* One decode step over a cache in either element format and either layout.
 *   fmt 0: k_cache/v_cache hold bf16 bits; fmt 1: E4M3 codes, the value of
 *          a code of KV head g being oracle_e4m3_value(code) * k_scale[g]
 *          (resp. v_scale[g]).
 *   block_table == NULL: packed caches [sum(max(seqlens,0)), n_kv, d], as in
 *          oracle_decode.  Otherwise paged caches [num_pages, page_size, n_kv, d]
 *          and block_table [B, max_blocks]: token t of sequence b is slot
 *          t % page_size of page block_table[b * max_blocks + t / page_size].
 * Returns -1 for bad shapes, a page index outside [0, num_pages) or a length
 * beyond max_blocks * page_size. */
int oracle_decode_general(const uint16_t *q, const void *k_cache, const void *v_cache, int fmt,
                          const float *k_scale, const float *v_scale, const int32_t *seqlens,
                          const int32_t *block_table, int max_blocks, int page_size, int num_pages,
                          double *out, int B, int h, int n_kv, int d, double scale, int n_threads) {
    if (!check_shape(B, h, n_kv, d) || (fmt != 0 && fmt != 1)) return -1;
    if (fmt == 1 && (!k_scale || !v_scale)) return -1;
    long *off = (long *)malloc(sizeof(long) * (size_t)B);
    if (!off) return -1;
    long acc = 0;
    for (int b = 0; b < B; ++b) { off[b] = acc; if (seqlens[b] > 0) acc += seqlens[b]; }
    if (block_table) {
        if (max_blocks <= 0 || page_size <= 0 || num_pages <= 0) { free(off); return -1; }
        for (int b = 0; b < B; ++b) {
            int L = seqlens[b];
            if (L > (long)max_blocks * page_size) { free(off); return -1; }
            for (int t = 0; t < L; t += page_size) {
                int page = block_table[(size_t)b * max_blocks + t / page_size];
                if (page < 0 || page >= num_pages) { free(off); return -1; }
            }
        }
    }
    job_t J = {0};
    J.kind = 2; J.q = q; J.kc = k_cache; J.vc = v_cache; J.fmt = fmt;
    J.k_scale = k_scale; J.v_scale = v_scale; J.seqlens = seqlens; J.offsets = off;
    J.block_table = block_table; J.max_blocks = max_blocks; J.page_size = page_size;
    J.out = out; J.B = B; J.h = h; J.n_kv = n_kv; J.d = d; J.scale = scale;
    J.n_units = B * h;
    int rc = run_job(&J, n_threads);
    free(off);
    return rc;
}

/* Chunked prefill over a paged bf16 cache, with the cache write.
 *   Same pages as oracle_decode_general: [num_pages, page_size, n_kv, d], token
 *   t of sequence b in slot t % page_size of page block_table[b][t / page_size].
 *   Sequence b holds past_lens[b] cached tokens; the chunk adds S_q tokens:
 *   q [B, S_q, h, d], k_new / v_new [B, S_q, n_kv, d].
 * Step 1 (the append; "Evolution of AI Attention Mechanisms", "MHA
 * Implementation": new K/V are concatenated after the past ones): row t of
 * k_new[b] / v_new[b] is copied to cache position past_lens[b] + t, for every
 * KV head.  k_pages / v_pages are updated in place.
 * Step 2: query row r of sequence b sits at position past_lens[b] + r and sees
 * keys at positions <= past_lens[b] + r (bottom-right causal), read back from
 * the updated pages.  out [B, S_q, h, d] fp64.
 * Returns -1 for bad shapes, a negative past length, a length past the block
 * table, or a page id outside [0, num_pages). */
int oracle_prefill_paged(const uint16_t *q, const uint16_t *k_new, const uint16_t *v_new,
                         uint16_t *k_pages, uint16_t *v_pages, const int32_t *block_table, int max_blocks,
                         int page_size, int num_pages, const int32_t *past_lens, double *out,
                         int B, int S_q, int h, int n_kv, int d, double scale, int n_threads) {
    (void)n_threads;
    if (!check_shape(B, h, n_kv, d) || S_q <= 0 || max_blocks <= 0 || page_size <= 0 || num_pages <= 0) return -1;
    for (int b = 0; b < B; ++b) {
        long total = (long)past_lens[b] + S_q;
        if (past_lens[b] < 0 || total > (long)max_blocks * page_size) return -1;
        for (long t = 0; t < total; t += page_size) {
            int page = block_table[(size_t)b * max_blocks + t / page_size];
            if (page < 0 || page >= num_pages) return -1;
        }
    }
    const size_t row = (size_t)n_kv * d;   /* elements of one cached token */
    /* step 1: the append */
    for (int b = 0; b < B; ++b)
        for (int t = 0; t < S_q; ++t) {
            long pos = (long)past_lens[b] + t;
            int page = block_table[(size_t)b * max_blocks + pos / page_size];
            size_t dst = ((size_t)page * page_size + (size_t)(pos % page_size)) * row;
            size_t src = ((size_t)b * S_q + t) * row;
            memcpy(k_pages + dst, k_new + src, sizeof(uint16_t) * row);
            memcpy(v_pages + dst, v_new + src, sizeof(uint16_t) * row);
        }
    /* step 2: attention over the gathered cache */
    int G = h / n_kv;
    for (int b = 0; b < B; ++b) {
        int total = past_lens[b] + S_q;
        double *kd = (double *)malloc(sizeof(double) * (size_t)total * d);
        double *vd = (double *)malloc(sizeof(double) * (size_t)total * d);
        double *qd = (double *)malloc(sizeof(double) * (size_t)S_q * d);
        double *o = (double *)malloc(sizeof(double) * (size_t)S_q * d);
        int *vis = (int *)malloc(sizeof(int) * (size_t)S_q);
        if (!kd || !vd || !qd || !o || !vis) { free(kd); free(vd); free(qd); free(o); free(vis); return -1; }
        for (int r = 0; r < S_q; ++r) vis[r] = past_lens[b] + r + 1;
        for (int g = 0; g < n_kv; ++g) {
            for (int t = 0; t < total; ++t) {
                int page = block_table[(size_t)b * max_blocks + t / page_size];
                size_t base = ((size_t)page * page_size + (size_t)(t % page_size)) * row + (size_t)g * d;
                for (int c = 0; c < d; ++c) {
                    kd[(size_t)t * d + c] = bf16_value(k_pages[base + c]);
                    vd[(size_t)t * d + c] = bf16_value(v_pages[base + c]);
                }
            }
            for (int i = g * G; i < (g + 1) * G; ++i) {
                for (int r = 0; r < S_q; ++r)
                    for (int c = 0; c < d; ++c)
                        qd[(size_t)r * d + c] = bf16_value(q[(((size_t)b * S_q + r) * h + i) * d + c]);
                if (attend_f64(qd, S_q, kd, vd, total, d, vis, scale, o, NULL)) {
                    free(kd); free(vd); free(qd); free(o); free(vis); return -1;
                }
                for (int r = 0; r < S_q; ++r)
                    memcpy(out + (((size_t)b * S_q + r) * h + i) * d, o + (size_t)r * d, sizeof(double) * (size_t)d);
            }
        }
        free(kd); free(vd); free(qd); free(o); free(vis);
    }
    return 0;
}

/*
 * Oracle for block-causal chunk attention -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the bench's CPU-baseline leg may load this file's library.
 * The product path (the CUDA library and its Python binding) never calls it, and this file shares
 * no code, header, table or constant with the CUDA path.
 *
 * What it computes is the plain definition of the attention the Wave Forcing DiT runs over the
 * mixed-noise wavefront:
 *   - within a chunk, attention is full; across chunks a query sees every earlier (cleaner) chunk
 *     and never a later (noisier) one  (KipQuest summary of arXiv 2611.00859, "The deep dive"
 *     transcript, paragraph on chunk-wise causal attention; project page, "01 The design gap",
 *     panel C "Directed live frontier");
 *   - each query chunk attends over all of that visible K/V with an ordinary softmax.
 * For query token t in chunk c and head h:
 *     s_j  = scale * sum_d q[t,h,d] * k[j,h,d]        for every key j whose chunk index <= c
 *     o    = sum_j softmax(s)_j * v[j,h,:]            (keys of chunks > c are excluded)
 *     lse  = log(sum_j exp(s_j))                      (natural log)
 * The mask is written out explicitly per key (chunk index of the key against chunk index of the
 * query); it is not the prefix shortcut the CUDA path uses, so the two formulations are
 * independent.  Inputs arrive as fp32 arrays holding bf16 values (exact); every sum is taken in
 * fp64; outputs are rounded to fp32.
 *
 * Layouts (row-major, contiguous):
 *   q    [T_q][H][D]   query rows of chunks num_ctx_chunks..num_chunks-1, in chunk order
 *   k, v [T_kv][H][D]  keys/values of all chunks in logical order (context first)
 *   out  [T_q][H][D]
 *   lse  [H][T_q]      (optional)
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const float *q, *k, *v;
    int H, D, T_q, T_kv, T_ctx;
    int num_chunks;
    const int32_t *chunk_offsets;
    const int32_t *key_chunk;     /* chunk index of every key, [T_kv] */
    double scale;
    /* work list: either all (row, head) pairs, or an explicit selection */
    int n_items;
    const int32_t *sel_rows, *sel_heads;   /* NULL => item i is (row = i / H, head = i % H) */
    float *out;                   /* full: [T_q][H][D]; selection: [n_items][D] */
    float *lse;                   /* full: [H][T_q];   selection: [n_items]    */
    int next_item;                /* shared work counter */
} job_t;

/* Chunk index of logical token t (chunk c holds tokens [offsets[c], offsets[c+1])). */
static int chunk_of_token(const int32_t *offsets, int num_chunks, int t) {
    for (int c = 0; c < num_chunks; ++c)
        if (t >= offsets[c] && t < offsets[c + 1]) return c;
    return -1;
}

/* Whether key j is visible to a query of chunk qc: keys of the same or an earlier chunk only. */
static int visible(const job_t *jb, int j, int qc) { return jb->key_chunk[j] <= qc; }

/* Key row j and value row j of head h. */
static const float *key_row(const job_t *jb, int j, int h) {
    return jb->k + ((size_t)j * jb->H + h) * jb->D;
}
static const float *value_row(const job_t *jb, int j, int h) {
    return jb->v + ((size_t)j * jb->H + h) * jb->D;
}

/* s[j] = scale * (q_r . k_j), each dot product summed in fp64 in d order.  Four visible keys are
 * summed side by side (four independent sums, each in the same order as alone); any key of a
 * later chunk is masked to -inf and its product is never formed.  Returns the largest logit. */
static double logits(const job_t *jb, const float *qr, int h, int qc, double *s) {
    const int D = jb->D, T_kv = jb->T_kv;
    double m = -INFINITY;
    int j = 0;
    while (j < T_kv) {
        if (j + 4 <= T_kv && visible(jb, j, qc) && visible(jb, j + 1, qc) &&
            visible(jb, j + 2, qc) && visible(jb, j + 3, qc)) {
            const float *k0 = key_row(jb, j, h), *k1 = key_row(jb, j + 1, h);
            const float *k2 = key_row(jb, j + 2, h), *k3 = key_row(jb, j + 3, h);
            double a0 = 0.0, a1 = 0.0, a2 = 0.0, a3 = 0.0;
            for (int d = 0; d < D; ++d) {
                const double x = (double)qr[d];
                a0 += x * (double)k0[d];
                a1 += x * (double)k1[d];
                a2 += x * (double)k2[d];
                a3 += x * (double)k3[d];
            }
            const double a[4] = {a0, a1, a2, a3};
            for (int i = 0; i < 4; ++i) {
                s[j + i] = jb->scale * a[i];
                if (s[j + i] > m) m = s[j + i];
            }
            j += 4;
            continue;
        }
        if (!visible(jb, j, qc)) { s[j] = -INFINITY; ++j; continue; }   /* later chunk: masked */
        const float *kr = key_row(jb, j, h);
        double acc = 0.0;
        for (int d = 0; d < D; ++d) {
            const double x = (double)qr[d];
            acc += x * (double)kr[d];
        }
        s[j] = jb->scale * acc;
        if (s[j] > m) m = s[j];
        ++j;
    }
    return m;
}

/* acc: D doubles of scratch. */
static void one_row(const job_t *jb, int r, int h, double *s, double *acc, float *o_out,
                    float *lse_out) {
    const int D = jb->D, T_kv = jb->T_kv;
    const int qc = chunk_of_token(jb->chunk_offsets, jb->num_chunks, jb->T_ctx + r);
    const float *qr = jb->q + ((size_t)r * jb->H + h) * D;
    const double m = logits(jb, qr, h, qc, s);
    double den = 0.0;
    for (int j = 0; j < T_kv; ++j) {
        if (!visible(jb, j, qc)) { s[j] = 0.0; continue; }
        s[j] = exp(s[j] - m);
        den += s[j];
    }
    /* o[d] = sum_j p_j v[j][d], every column summed over ascending j */
    for (int d = 0; d < D; ++d) acc[d] = 0.0;
    for (int j = 0; j < T_kv; ++j) {
        if (s[j] == 0.0) continue;
        const float *vr = value_row(jb, j, h);
        const double p = s[j];
        for (int d = 0; d < D; ++d) acc[d] += p * (double)vr[d];
    }
    for (int d = 0; d < D; ++d) o_out[d] = (float)(acc[d] / den);
    if (lse_out) *lse_out = (float)(m + log(den));
}

static void *worker(void *arg) {
    job_t *jb = (job_t *)arg;
    double *s = (double *)malloc(sizeof(double) * (size_t)(jb->T_kv > 0 ? jb->T_kv : 1));
    double *acc = (double *)malloc(sizeof(double) * (size_t)jb->D);
    if (!s || !acc) { free(s); free(acc); return (void *)1; }
    for (;;) {
        int i = __atomic_fetch_add(&jb->next_item, 1, __ATOMIC_RELAXED);
        if (i >= jb->n_items) break;
        int r, h;
        float *o, *l;
        if (jb->sel_rows) {
            r = jb->sel_rows[i];
            h = jb->sel_heads[i];
            o = jb->out + (size_t)i * jb->D;
            l = jb->lse ? jb->lse + i : NULL;
        } else {
            r = i / jb->H;
            h = i % jb->H;
            o = jb->out + ((size_t)r * jb->H + h) * jb->D;
            l = jb->lse ? jb->lse + (size_t)h * jb->T_q + r : NULL;
        }
        one_row(jb, r, h, s, acc, o, l);
    }
    free(s);
    free(acc);
    return NULL;
}

static int run(job_t *jb, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    pthread_t th[256];
    int started = 0, rc = 0;
    for (int t = 0; t < nthreads; ++t) {
        if (pthread_create(&th[t], NULL, worker, jb) != 0) { rc = 3; break; }
        ++started;
    }
    for (int t = 0; t < started; ++t) {
        void *ret = NULL;
        pthread_join(th[t], &ret);
        if (ret) rc = 4;
    }
    return rc;
}

static int setup(job_t *jb, const float *q, const float *k, const float *v, int H, int D,
                 int num_chunks, int num_ctx_chunks, const int32_t *chunk_offsets, double scale,
                 int32_t **key_chunk_out) {
    if (!q || !k || !v || !chunk_offsets || H < 1 || D < 1 || num_chunks < 1 ||
        num_ctx_chunks < 0 || num_ctx_chunks >= num_chunks || chunk_offsets[0] != 0)
        return 1;
    for (int c = 0; c < num_chunks; ++c)
        if (chunk_offsets[c + 1] < chunk_offsets[c]) return 1;
    memset(jb, 0, sizeof(*jb));
    jb->q = q; jb->k = k; jb->v = v; jb->H = H; jb->D = D;
    jb->num_chunks = num_chunks;
    jb->chunk_offsets = chunk_offsets;
    jb->T_kv = chunk_offsets[num_chunks];
    jb->T_ctx = chunk_offsets[num_ctx_chunks];
    jb->T_q = jb->T_kv - jb->T_ctx;
    jb->scale = scale;
    int32_t *kc = (int32_t *)malloc(sizeof(int32_t) * (size_t)(jb->T_kv > 0 ? jb->T_kv : 1));
    if (!kc) return 2;
    for (int j = 0; j < jb->T_kv; ++j) kc[j] = chunk_of_token(chunk_offsets, num_chunks, j);
    jb->key_chunk = kc;
    *key_chunk_out = kc;
    return 0;
}

/* Every (row, head) of the wavefront.  Returns 0 on success. */
int oracle_attention(const float *q, const float *k, const float *v, int H, int D, int num_chunks,
                     int num_ctx_chunks, const int32_t *chunk_offsets, double scale, float *out,
                     float *lse, int nthreads) {
    job_t jb;
    int32_t *kc = NULL;
    int rc = setup(&jb, q, k, v, H, D, num_chunks, num_ctx_chunks, chunk_offsets, scale, &kc);
    if (rc) return rc;
    if (!out) { free(kc); return 1; }
    jb.n_items = jb.T_q * H;
    jb.out = out;
    jb.lse = lse;
    rc = run(&jb, nthreads);
    free(kc);
    return rc;
}

/* A selection of (row, head) pairs: out_sel [n_sel][D], lse_sel [n_sel] (optional). */
int oracle_attention_rows(const float *q, const float *k, const float *v, int H, int D,
                          int num_chunks, int num_ctx_chunks, const int32_t *chunk_offsets,
                          double scale, const int32_t *rows, const int32_t *heads, int n_sel,
                          float *out_sel, float *lse_sel, int nthreads) {
    job_t jb;
    int32_t *kc = NULL;
    int rc = setup(&jb, q, k, v, H, D, num_chunks, num_ctx_chunks, chunk_offsets, scale, &kc);
    if (rc) return rc;
    if (!rows || !heads || !out_sel || n_sel < 0) { free(kc); return 1; }
    for (int i = 0; i < n_sel; ++i)
        if (rows[i] < 0 || rows[i] >= jb.T_q || heads[i] < 0 || heads[i] >= H) { free(kc); return 1; }
    jb.n_items = n_sel;
    jb.sel_rows = rows;
    jb.sel_heads = heads;
    jb.out = out_sel;
    jb.lse = lse_sel;
    rc = run(&jb, nthreads);
    free(kc);
    return rc;
}

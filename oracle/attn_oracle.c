/*
 * attn_oracle.c -- plain fp64 CPU attention forward (threaded with pthreads).
 *
 * TEST INFRASTRUCTURE ONLY.  Built as liboracle_attn.so and called through
 * ctypes by the test suite and by bench.py's CPU-baseline / reference legs.
 * It shares no code with the CUDA library and is never linked into it.
 *
 * What it computes (written from the definition):
 *   "带你了解Attention,从MHA到DeepSeek", section 1.2: score = q.k,
 *   weights = softmax(score / sqrt(d_k)), output = sum of weights * v.
 *   "GQA和MLA详解", sections 1-2: causal mask; G query heads share one K/V
 *   head (query head h reads kv head h / G, as repeat_interleave does).
 *
 * For each (b, h, i):
 *   n   = visible keys (all skv[b] keys; causal: j <= i + skv[b] - Sq)
 *   s_j = scale * sum_t q[t] k_j[t]              for j < n
 *   m   = max_j s_j;  e_j = exp(s_j - m);  l = sum_j e_j
 *   out = sum_j e_j v_j / l;  lse = m + log(l)   (n == 0: out = 0, lse = -inf)
 *
 * Inputs are float (the exact bf16/fp16 values the GPU gets, upcast); all
 * arithmetic is double.  Tensors are addressed with element strides
 * (b, h, s; the innermost stride is 1), so a latent cache [B, S, 576] and its
 * first-512-column value view can be passed without copies.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const float *q, *k, *v;
    double *out, *lse;
    int B, Hq, Hkv, Sq, dk, dv, causal;
    const int *skv;
    int64_t qsb, qsh, qss, ksb, ksh, kss, vsb, vsh, vss;
    double scale;
    const int *rows; /* optional list of (b, h) pairs; NULL = all */
    int nrows;
    int next;        /* work counter */
    pthread_mutex_t mu;
} job_t;

static int visible(int i, int Sq, int L, int causal) {
    if (!causal) return L;
    int n = i + L - Sq + 1;
    if (n < 0) n = 0;
    if (n > L) n = L;
    return n;
}

static void do_pair(job_t *J, int b, int h, double *s) {
    const int G = J->Hq / J->Hkv;
    const int L = J->skv[b];
    const float *qb = J->q + b * J->qsb + h * J->qsh;
    const float *kb = J->k + b * J->ksb + (h / G) * J->ksh;
    const float *vb = J->v + b * J->vsb + (h / G) * J->vsh;
    for (int i = 0; i < J->Sq; ++i) {
        double *o = J->out + (((int64_t)b * J->Hq + h) * J->Sq + i) * J->dv;
        double *ls = J->lse + ((int64_t)b * J->Hq + h) * J->Sq + i;
        int n = visible(i, J->Sq, L, J->causal);
        for (int c = 0; c < J->dv; ++c) o[c] = 0.0;
        if (n == 0) { *ls = -INFINITY; continue; }
        const float *qi = qb + (int64_t)i * J->qss;
        double m = -INFINITY;
        for (int j = 0; j < n; ++j) {
            const float *kj = kb + (int64_t)j * J->kss;
            double acc = 0.0;
            for (int t = 0; t < J->dk; ++t) acc += (double)qi[t] * (double)kj[t];
            s[j] = J->scale * acc;
            if (s[j] > m) m = s[j];
        }
        double l = 0.0;
        for (int j = 0; j < n; ++j) {
            double e = exp(s[j] - m);
            l += e;
            const float *vj = vb + (int64_t)j * J->vss;
            for (int c = 0; c < J->dv; ++c) o[c] += e * (double)vj[c];
        }
        for (int c = 0; c < J->dv; ++c) o[c] /= l;
        *ls = m + log(l);
    }
}

static void *worker(void *arg) {
    job_t *J = (job_t *)arg;
    int maxL = 1;
    for (int b = 0; b < J->B; ++b) if (J->skv[b] > maxL) maxL = J->skv[b];
    double *s = (double *)malloc(sizeof(double) * (size_t)maxL);
    if (!s) return NULL;
    const int total = J->rows ? J->nrows : J->B * J->Hq;
    for (;;) {
        pthread_mutex_lock(&J->mu);
        int w = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (w >= total) break;
        int b, h;
        if (J->rows) { b = J->rows[2 * w]; h = J->rows[2 * w + 1]; }
        else { b = w / J->Hq; h = w % J->Hq; }
        do_pair(J, b, h, s);
    }
    free(s);
    return NULL;
}

/*
 * Returns 0 on success, -1 on bad arguments.
 * out: [B, Hq, Sq, dv] double; lse: [B, Hq, Sq] double (rows not listed in
 * `rows` are left untouched).  nthreads <= 0 means 1.
 */
int oracle_attn_fwd(const float *q, const float *k, const float *v,
                    double *out, double *lse,
                    int B, int Hq, int Hkv, int Sq, const int *skv,
                    int dk, int dv,
                    int64_t qsb, int64_t qsh, int64_t qss,
                    int64_t ksb, int64_t ksh, int64_t kss,
                    int64_t vsb, int64_t vsh, int64_t vss,
                    double scale, int causal, int nthreads,
                    const int *rows, int nrows) {
    if (!q || !k || !v || !out || !lse || !skv) return -1;
    if (B <= 0 || Hq <= 0 || Hkv <= 0 || Sq <= 0 || dk <= 0 || dv <= 0) return -1;
    if (Hq % Hkv) return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.out = out; J.lse = lse;
    J.B = B; J.Hq = Hq; J.Hkv = Hkv; J.Sq = Sq; J.dk = dk; J.dv = dv;
    J.causal = causal; J.skv = skv;
    J.qsb = qsb; J.qsh = qsh; J.qss = qss;
    J.ksb = ksb; J.ksh = ksh; J.kss = kss;
    J.vsb = vsb; J.vsh = vsh; J.vss = vss;
    J.scale = scale; J.rows = rows; J.nrows = nrows;
    pthread_mutex_init(&J.mu, NULL);
    if (nthreads <= 0) nthreads = 1;
    if (nthreads > 512) nthreads = 512;
    pthread_t th[512];
    int started = 0;
    for (int t = 0; t < nthreads; ++t)
        if (pthread_create(&th[t], NULL, worker, &J) == 0) ++started;
    if (started == 0) worker(&J);
    for (int t = 0; t < started; ++t) pthread_join(th[t], NULL);
    pthread_mutex_destroy(&J.mu);
    return 0;
}

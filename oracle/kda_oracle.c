/*
 * CPU oracle for the Kimi Delta Attention (KDA) forward pass.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the library's product path links,
 * loads or calls this file; only the tests, the smoke check and the
 * benchmark's CPU-baseline leg do.  It shares no code with the CUDA path.
 *
 * What it computes: the KDA recurrence, per head and token t,
 *
 *   S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
 *   o_t = scale * S_t^T q_t,
 *
 * in fp64 on the exact input values (bf16 and fp32 inputs arrive as fp32,
 * which holds both exactly).  The per-channel decay Diag(alpha_t) and the
 * beta-scaled delta rule are the key equation of "Kimi Delta Attention: The
 * Linear Attention Behind Kimi K2 and Qwen3" (§TL;DR, and the order of the
 * operations stated in prose in §How Kimi Delta Attention works step by
 * step); the factor (I - beta k k^T) is the forgetting form of the delta rule
 * in "KDA Technical Deep Dive", §From attention to recurrent state.  The
 * product is evaluated in its expanded form, which needs no dk x dk matrix:
 * with S the dk x dv state (rows = key channels),
 *
 *   S~  = Diag(alpha_t) S,  alpha_t = exp(log_alpha_t)     (decay)
 *   e   = beta_t (v_t - S~^T k_t)                           (delta-rule error)
 *   S   = S~ + k_t e^T  = (I - beta_t k_t k_t^T) S~ + beta_t k_t v_t^T
 *   o_t = scale * S^T q_t                                   (read after the write)
 *
 * The pages write the state as a (d_v, d_k) matrix that maps keys to values;
 * this file stores its transpose (dk x dv, value axis contiguous), so the
 * prediction is S~^T k and the per-channel decay scales rows.  `scale` is the
 * 1/sqrt(d_k) query scaling of the KDA page's read unless the caller passes
 * another value.
 *
 * Layouts (row-major, contiguous): q, k, log_alpha [B,T,H,dk] fp32;
 * v [B,T,H,dv] fp32; beta [B,T,H] fp32; s0 [B,H,dk,dv] fp64 or NULL (zeros);
 * out [B,T,H,dv] fp64; s_final [B,H,dk,dv] fp64 or NULL.  s_final may alias
 * s0.  `nthreads` <= 0 uses one thread per online core.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const float *q, *k, *v, *log_alpha, *beta;
    const double *s0;
    double *out, *s_final;
    int B, T, H, dk, dv;
    double scale;
    int next_head;            /* work counter, guarded by lock */
    pthread_mutex_t lock;
} oracle_job;

static void run_one_head(const oracle_job *j, int bh, double *S, double *p, double *e)
{
    const int b = bh / j->H, h = bh % j->H;
    const int dk = j->dk, dv = j->dv, H = j->H;
    if (j->s0)
        memcpy(S, j->s0 + (size_t)bh * dk * dv, sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);

    for (int t = 0; t < j->T; ++t) {
        const size_t tok = (size_t)b * j->T + t;            /* token index in [B,T] */
        const float *qt = j->q + (tok * H + h) * dk;
        const float *kt = j->k + (tok * H + h) * dk;
        const float *vt = j->v + (tok * H + h) * dv;
        const float *lat = j->log_alpha + (tok * H + h) * dk;
        const double bt = (double)j->beta[tok * H + h];
        double *ot = j->out + (tok * H + h) * dv;

        /* S~ = Diag(alpha_t) S: key channel c (row c) scaled by exp(log_alpha_t[c]) */
        for (int c = 0; c < dk; ++c) {
            const double a = exp((double)lat[c]);
            double *row = S + (size_t)c * dv;
            for (int x = 0; x < dv; ++x) row[x] *= a;
        }
        /* p = S~^T k_t: the value the decayed state maps k_t to */
        for (int x = 0; x < dv; ++x) p[x] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double kc = (double)kt[c];
            const double *row = S + (size_t)c * dv;
            for (int x = 0; x < dv; ++x) p[x] += row[x] * kc;
        }
        /* e = beta_t (v_t - p) */
        for (int x = 0; x < dv; ++x) e[x] = bt * ((double)vt[x] - p[x]);
        /* S_t = S~ + k_t e^T = (I - beta_t k_t k_t^T) S~ + beta_t k_t v_t^T */
        for (int c = 0; c < dk; ++c) {
            const double kc = (double)kt[c];
            double *row = S + (size_t)c * dv;
            for (int x = 0; x < dv; ++x) row[x] += kc * e[x];
        }
        /* o_t = scale * S_t^T q_t (the state after this token's write) */
        for (int x = 0; x < dv; ++x) ot[x] = 0.0;
        for (int c = 0; c < dk; ++c) {
            const double qc = (double)qt[c];
            const double *row = S + (size_t)c * dv;
            for (int x = 0; x < dv; ++x) ot[x] += row[x] * qc;
        }
        for (int x = 0; x < dv; ++x) ot[x] *= j->scale;
    }
    if (j->s_final)
        memcpy(j->s_final + (size_t)bh * dk * dv, S, sizeof(double) * (size_t)dk * dv);
}

static void *worker(void *arg)
{
    oracle_job *j = (oracle_job *)arg;
    const size_t n = (size_t)j->dk * j->dv + 2 * (size_t)j->dv;
    double *buf = (double *)malloc(sizeof(double) * n);
    if (!buf) return (void *)1;
    double *S = buf, *p = buf + (size_t)j->dk * j->dv, *e = p + j->dv;
    for (;;) {
        pthread_mutex_lock(&j->lock);
        const int bh = j->next_head++;
        pthread_mutex_unlock(&j->lock);
        if (bh >= j->B * j->H) break;
        run_one_head(j, bh, S, p, e);
    }
    free(buf);
    return NULL;
}

/* Returns 0 on success, -1 on a bad argument, -2 on an allocation or thread failure. */
int kda_oracle_forward(const float *q, const float *k, const float *v,
                       const float *log_alpha, const float *beta,
                       const double *s0, double *out, double *s_final,
                       int B, int T, int H, int dk, int dv, double scale, int nthreads)
{
    if (!q || !k || !v || !log_alpha || !beta || (!out && T > 0)) return -1;
    if (B <= 0 || H <= 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
    oracle_job j;
    j.q = q; j.k = k; j.v = v; j.log_alpha = log_alpha; j.beta = beta;
    j.s0 = s0; j.out = out; j.s_final = s_final;
    j.B = B; j.T = T; j.H = H; j.dk = dk; j.dv = dv; j.scale = scale;
    j.next_head = 0;
    pthread_mutex_init(&j.lock, NULL);
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads > B * H) nthreads = B * H;
    if (nthreads < 1) nthreads = 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * (size_t)nthreads);
    if (!th) return -2;
    int started = 0, rc = 0;
    for (; started < nthreads; ++started)
        if (pthread_create(&th[started], NULL, worker, &j) != 0) break;
    if (started == 0) {               /* no thread could start: run inline */
        if (worker(&j) != NULL) rc = -2;
    }
    for (int i = 0; i < started; ++i) {
        void *r = NULL;
        pthread_join(th[i], &r);
        if (r != NULL) rc = -2;
    }
    free(th);
    pthread_mutex_destroy(&j.lock);
    return rc;
}

/* Number of threads kda_oracle_forward uses for B*H heads with nthreads <= 0. */
int kda_oracle_default_threads(void) { return (int)sysconf(_SC_NPROCESSORS_ONLN); }

/*
 * Gated delta-rule oracle: plain fp64 token-by-token recurrence on the CPU.
 *
 * TEST INFRASTRUCTURE ONLY. This file is the correctness reference that the
 * CUDA library is checked against. Only the tests, the smoke check and the
 * benchmark's CPU-baseline leg may load it. It shares no code, header, table
 * or helper with the CUDA library, and the CUDA library never calls it.
 *
 * What it computes (the plain definition, not an algorithm transcript):
 *
 *   For every (batch row b, value head h), with key head hk = h / (Hv/Hk):
 *     S <- h0[b,h]                      (Dk x Dv, the "K x V state"; zeros if h0 is NULL)
 *     for t = 0 .. T-1:
 *       S <- diag(exp(g_t)) S           decay first (scalar per head, or per key channel)
 *       p <- S^T k_t                    the memory's prediction for key k_t
 *       S <- S + beta_t k_t (v_t - p)^T the delta correction
 *       o_t <- S^T q_t                  readout after the update, scale 1
 *     hT[b,h] <- S
 *
 * Sources:
 *   - NextTransformer, "Source notes", section "Linear attention": the state S
 *     is K x V; row gdn gives S <- alpha (I - beta k k^T) S + beta k v^T with a
 *     scalar per-head decay applied before the delta update; row kda gives the
 *     feature-wise (per key channel) decay before the delta update; row
 *     deltanet gives S <- S + k[beta(v - k^T S)]^T and the readout y = q^T S.
 *   - Same page, "Backend and numerical limits": explicit scale = 1; an FP64
 *     recurrent scan is the correctness reference.
 *   - Frontier-model atlas, item 03 (Gated DeltaNet): state decay, memory
 *     prediction, delta correction, recurrent read, in that order.
 *   - Frontier-model atlas, item 08: 16 key heads shared by 48 value heads
 *     (grouped value heads); value head h reads key head h / (Hv/Hk).
 *
 * Note that alpha (I - beta k k^T) S + beta k v^T = S' + beta k (v - S'^T k)^T
 * with S' = alpha S, which is the form written above.
 *
 * Layouts (row-major, contiguous, all fp64):
 *   q, k  [B, T, Hk, Dk]      v, o  [B, T, Hv, Dv]
 *   g     [B, T, Hv] (gate_mode 0, scalar) or [B, T, Hv, Dk] (gate_mode 1, per channel)
 *   beta  [B, T, Hv]          h0, hT [B, Hv, Dk, Dv]   (either may be NULL)
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

typedef struct {
    const double *q, *k, *v, *g, *beta, *h0;
    double *o, *hT;
    int B, T, Hk, Hv, Dk, Dv, gate_mode;
    long next_unit;        /* shared work counter, guarded by lock */
    pthread_mutex_t lock;
} job_t;

static void run_unit(const job_t *J, long unit, double *S, double *p)
{
    const int B = J->B, T = J->T, Hk = J->Hk, Hv = J->Hv, Dk = J->Dk, Dv = J->Dv;
    const int b = (int)(unit / Hv), h = (int)(unit % Hv);
    const int hk = h / (Hv / Hk);
    (void)B;

    if (J->h0)
        memcpy(S, J->h0 + ((size_t)b * Hv + h) * Dk * Dv, sizeof(double) * Dk * Dv);
    else
        memset(S, 0, sizeof(double) * Dk * Dv);

    for (int t = 0; t < T; ++t) {
        const double *kt = J->k + (((size_t)b * T + t) * Hk + hk) * Dk;
        const double *qt = J->q + (((size_t)b * T + t) * Hk + hk) * Dk;
        const double *vt = J->v + (((size_t)b * T + t) * Hv + h) * Dv;
        const double bt = J->beta[((size_t)b * T + t) * Hv + h];
        double *ot = J->o ? J->o + (((size_t)b * T + t) * Hv + h) * Dv : NULL;

        /* decay: S <- diag(exp(g_t)) S */
        for (int c = 0; c < Dk; ++c) {
            double a;
            if (J->gate_mode == 0)
                a = exp(J->g[((size_t)b * T + t) * Hv + h]);
            else
                a = exp(J->g[(((size_t)b * T + t) * Hv + h) * Dk + c]);
            for (int j = 0; j < Dv; ++j) S[(size_t)c * Dv + j] *= a;
        }
        /* prediction: p = S^T k_t */
        for (int j = 0; j < Dv; ++j) p[j] = 0.0;
        for (int c = 0; c < Dk; ++c)
            for (int j = 0; j < Dv; ++j) p[j] += S[(size_t)c * Dv + j] * kt[c];
        /* correction: S <- S + beta_t k_t (v_t - p)^T */
        for (int c = 0; c < Dk; ++c) {
            const double bk = bt * kt[c];
            for (int j = 0; j < Dv; ++j) S[(size_t)c * Dv + j] += bk * (vt[j] - p[j]);
        }
        /* readout: o_t = S^T q_t */
        if (ot) {
            for (int j = 0; j < Dv; ++j) ot[j] = 0.0;
            for (int c = 0; c < Dk; ++c)
                for (int j = 0; j < Dv; ++j) ot[j] += S[(size_t)c * Dv + j] * qt[c];
        }
    }
    if (J->hT)
        memcpy(J->hT + ((size_t)b * Hv + h) * Dk * Dv, S, sizeof(double) * Dk * Dv);
}

static void *worker(void *arg)
{
    job_t *J = (job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * (size_t)J->Dk * J->Dv);
    double *p = (double *)malloc(sizeof(double) * (size_t)J->Dv);
    const long units = (long)J->B * J->Hv;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        long u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= units) break;
        run_unit(J, u, S, p);
    }
    free(S);
    free(p);
    return NULL;
}

/* Returns 0 on success, -1 on bad arguments. nthreads <= 0 uses every online core. */
int gdr_oracle_recurrent(const double *q, const double *k, const double *v, const double *g,
                         const double *beta, const double *h0, double *o, double *hT,
                         int B, int T, int Hk, int Hv, int Dk, int Dv, int gate_mode, int nthreads)
{
    if (B <= 0 || T < 0 || Hk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0) return -1;
    if (Hv % Hk != 0 || (gate_mode != 0 && gate_mode != 1)) return -1;
    if (T > 0 && (!q || !k || !v || !g || !beta)) return -1;

    job_t J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.h0 = h0; J.o = o; J.hT = hT;
    J.B = B; J.T = T; J.Hk = Hk; J.Hv = Hv; J.Dk = Dk; J.Dv = Dv; J.gate_mode = gate_mode;
    J.next_unit = 0;
    pthread_mutex_init(&J.lock, NULL);

    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    const long units = (long)B * Hv;
    if (nthreads > units) nthreads = (int)units;

    if (nthreads == 1) {
        worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
        for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/* Number of threads gdr_oracle_recurrent uses for a given request (for reporting). */
int gdr_oracle_threads(int nthreads, long units)
{
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > units) nthreads = (int)units;
    return nthreads;
}

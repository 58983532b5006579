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

/*
 * Backward of the recurrence above (the adjoint of the token loop, fp64).
 *
 * Given the upstream gradients do = dL/do [B, T, Hv, Dv] and dhT = dL/dhT
 * [B, Hv, Dk, Dv] (NULL: zero), returns dL/dq, dL/dk [B, T, Hk, Dk], dL/dv
 * [B, T, Hv, Dv], dL/dg (the layout of g), dL/dbeta [B, T, Hv] and dL/dh0
 * [B, Hv, Dk, Dv]. It runs the forward keeping every state, then reverses each
 * step of the token loop:
 *
 *   forward step t:  Sb = diag(a_t) S,  a_t = exp(g_t);  p = Sb^T k;  e = v - p;
 *                    u = beta e;  S' = Sb + k u^T;  o = S'^T q
 *   reverse step t:  dS += q do^T;  dq = S' do;  du = dS^T k;  dk = dS u;
 *                    dbeta = du . e;  dv = beta du;  dp = -beta du;
 *                    dSb = dS + k dp^T;  dk += Sb dp;
 *                    dg_c = sum_j dSb[c][j] Sb[c][j]  (summed over c for a scalar gate);
 *                    dS <- diag(a_t) dSb
 *
 * dq and dk sum over the value heads that share a key head, so the work is
 * split by (batch row, key head). Returns 0, or -1 on bad arguments.
 */
typedef struct {
    const double *q, *k, *v, *g, *beta, *h0, *dout, *dhT;
    double *dq, *dk, *dv, *dg, *dbeta, *dh0;
    int B, T, Hk, Hv, Dk, Dv, gate_mode;
    long next_unit;
    pthread_mutex_t lock;
} bjob_t;

static void run_bwd_unit(const bjob_t *J, int b, int h, double *states, double *S, double *dS, double *Sb,
                         double *p, double *e, double *du)
{
    const int T = J->T, Hk = J->Hk, Hv = J->Hv, Dk = J->Dk, Dv = J->Dv;
    const int hk = h / (Hv / Hk);
    const size_t SZ = (size_t)Dk * Dv;
    if (J->h0)
        memcpy(S, J->h0 + ((size_t)b * Hv + h) * SZ, sizeof(double) * SZ);
    else
        memset(S, 0, sizeof(double) * SZ);
#define A_T(t, c) (J->gate_mode == 0 ? exp(J->g[((size_t)b * T + (t)) * Hv + h]) \
                                     : exp(J->g[(((size_t)b * T + (t)) * Hv + h) * Dk + (c)]))
    /* forward, keeping the state before every token */
    for (int t = 0; t < T; ++t) {
        const double *kt = J->k + (((size_t)b * T + t) * Hk + hk) * Dk;
        const double *vt = J->v + (((size_t)b * T + t) * Hv + h) * Dv;
        const double bt = J->beta[((size_t)b * T + t) * Hv + h];
        memcpy(states + (size_t)t * SZ, S, sizeof(double) * SZ);
        for (int c = 0; c < Dk; ++c) {
            const double a = A_T(t, c);
            for (int j = 0; j < Dv; ++j) S[(size_t)c * Dv + j] *= a;
        }
        for (int j = 0; j < Dv; ++j) p[j] = 0.0;
        for (int c = 0; c < Dk; ++c)
            for (int j = 0; j < Dv; ++j) p[j] += S[(size_t)c * Dv + j] * kt[c];
        for (int c = 0; c < Dk; ++c)
            for (int j = 0; j < Dv; ++j) S[(size_t)c * Dv + j] += bt * kt[c] * (vt[j] - p[j]);
    }
    /* reverse */
    if (J->dhT)
        memcpy(dS, J->dhT + ((size_t)b * Hv + h) * SZ, sizeof(double) * SZ);
    else
        memset(dS, 0, sizeof(double) * SZ);
    for (int t = T - 1; t >= 0; --t) {
        const double *kt = J->k + (((size_t)b * T + t) * Hk + hk) * Dk;
        const double *qt = J->q + (((size_t)b * T + t) * Hk + hk) * Dk;
        const double *vt = J->v + (((size_t)b * T + t) * Hv + h) * Dv;
        const double *dot = J->dout + (((size_t)b * T + t) * Hv + h) * Dv;
        const double bt = J->beta[((size_t)b * T + t) * Hv + h];
        double *dqt = J->dq + (((size_t)b * T + t) * Hk + hk) * Dk;
        double *dkt = J->dk + (((size_t)b * T + t) * Hk + hk) * Dk;
        double *dvt = J->dv + (((size_t)b * T + t) * Hv + h) * Dv;
        const double *Sp = states + (size_t)t * SZ;
        /* recompute this step's quantities */
        for (int c = 0; c < Dk; ++c) {
            const double a = A_T(t, c);
            for (int j = 0; j < Dv; ++j) Sb[(size_t)c * Dv + j] = a * Sp[(size_t)c * Dv + j];
        }
        for (int j = 0; j < Dv; ++j) p[j] = 0.0;
        for (int c = 0; c < Dk; ++c)
            for (int j = 0; j < Dv; ++j) p[j] += Sb[(size_t)c * Dv + j] * kt[c];
        for (int j = 0; j < Dv; ++j) e[j] = vt[j] - p[j];
        /* o = S'^T q with S' = Sb + k (beta e)^T */
        for (int c = 0; c < Dk; ++c)
            for (int j = 0; j < Dv; ++j) dS[(size_t)c * Dv + j] += qt[c] * dot[j];
        for (int c = 0; c < Dk; ++c) {
            double s = 0.0;
            for (int j = 0; j < Dv; ++j) s += (Sb[(size_t)c * Dv + j] + kt[c] * bt * e[j]) * dot[j];
            dqt[c] += s;
        }
        /* S' = Sb + k u^T */
        for (int j = 0; j < Dv; ++j) du[j] = 0.0;
        for (int c = 0; c < Dk; ++c)
            for (int j = 0; j < Dv; ++j) du[j] += dS[(size_t)c * Dv + j] * kt[c];
        for (int c = 0; c < Dk; ++c) {
            double s = 0.0;
            for (int j = 0; j < Dv; ++j) s += dS[(size_t)c * Dv + j] * bt * e[j];
            dkt[c] += s;
        }
        /* u = beta e, e = v - p */
        double db = 0.0;
        for (int j = 0; j < Dv; ++j) db += du[j] * e[j];
        J->dbeta[((size_t)b * T + t) * Hv + h] = db;
        for (int j = 0; j < Dv; ++j) dvt[j] = bt * du[j];
        /* p = Sb^T k: dSb = dS + k dp^T, dk += Sb dp, dp = -beta du */
        for (int c = 0; c < Dk; ++c) {
            double s = 0.0;
            for (int j = 0; j < Dv; ++j) {
                const double dp = -bt * du[j];
                dS[(size_t)c * Dv + j] += kt[c] * dp;
                s += Sb[(size_t)c * Dv + j] * dp;
            }
            dkt[c] += s;
        }
        /* Sb = diag(a) S_prev */
        double dgs = 0.0;
        for (int c = 0; c < Dk; ++c) {
            double s = 0.0;
            for (int j = 0; j < Dv; ++j) s += dS[(size_t)c * Dv + j] * Sb[(size_t)c * Dv + j];
            if (J->gate_mode == 1)
                J->dg[(((size_t)b * T + t) * Hv + h) * Dk + c] = s;
            else
                dgs += s;
            const double a = A_T(t, c);
            for (int j = 0; j < Dv; ++j) dS[(size_t)c * Dv + j] *= a;
        }
        if (J->gate_mode == 0) J->dg[((size_t)b * T + t) * Hv + h] = dgs;
    }
#undef A_T
    memcpy(J->dh0 + ((size_t)b * Hv + h) * SZ, dS, sizeof(double) * SZ);
}

static void *bwd_worker(void *arg)
{
    bjob_t *J = (bjob_t *)arg;
    const size_t SZ = (size_t)J->Dk * J->Dv;
    double *states = (double *)malloc(sizeof(double) * SZ * (size_t)(J->T > 0 ? J->T : 1));
    double *S = (double *)malloc(sizeof(double) * SZ), *dS = (double *)malloc(sizeof(double) * SZ);
    double *Sb = (double *)malloc(sizeof(double) * SZ);
    double *p = (double *)malloc(sizeof(double) * J->Dv), *e = (double *)malloc(sizeof(double) * J->Dv);
    double *du = (double *)malloc(sizeof(double) * J->Dv);
    const long units = (long)J->B * J->Hk;
    const int grp = J->Hv / J->Hk;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        long u = J->next_unit++;
        pthread_mutex_unlock(&J->lock);
        if (u >= units) break;
        const int b = (int)(u / J->Hk), hk = (int)(u % J->Hk);
        for (int i = 0; i < grp; ++i) run_bwd_unit(J, b, hk * grp + i, states, S, dS, Sb, p, e, du);
    }
    free(states); free(S); free(dS); free(Sb); free(p); free(e); free(du);
    return NULL;
}

int gdr_oracle_backward(const double *q, const double *k, const double *v, const double *g, const double *beta,
                        const double *h0, const double *dout, const double *dhT, double *dq, double *dk,
                        double *dv, double *dg, double *dbeta, double *dh0, int B, int T, int Hk, int Hv, int Dk,
                        int Dv, int gate_mode, int nthreads)
{
    if (B <= 0 || T < 0 || Hk <= 0 || Hv <= 0 || Dk <= 0 || Dv <= 0) return -1;
    if (Hv % Hk != 0 || (gate_mode != 0 && gate_mode != 1)) return -1;
    if (T > 0 && (!q || !k || !v || !g || !beta || !dout)) return -1;
    if (!dq || !dk || !dv || !dg || !dbeta || !dh0) return -1;
    bjob_t J;
    J.q = q; J.k = k; J.v = v; J.g = g; J.beta = beta; J.h0 = h0; J.dout = dout; J.dhT = dhT;
    J.dq = dq; J.dk = dk; J.dv = dv; J.dg = dg; J.dbeta = dbeta; J.dh0 = dh0;
    J.B = B; J.T = T; J.Hk = Hk; J.Hv = Hv; J.Dk = Dk; J.Dv = Dv; J.gate_mode = gate_mode;
    J.next_unit = 0;
    memset(dq, 0, sizeof(double) * (size_t)B * T * Hk * Dk);
    memset(dk, 0, sizeof(double) * (size_t)B * T * Hk * Dk);
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    const long units = (long)B * Hk;
    if (nthreads > units) nthreads = (int)units;
    if (nthreads == 1) {
        bwd_worker(&J);
    } else {
        pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
        for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, bwd_worker, &J);
        for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
        free(th);
    }
    pthread_mutex_destroy(&J.lock);
    return 0;
}

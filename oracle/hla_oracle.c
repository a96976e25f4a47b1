/*
 * fp64 CPU oracle for the strictly causal masked Higher-order Linear Attention
 * forward.  TEST INFRASTRUCTURE ONLY: the tests, the package's smoke check and
 * the bench's CPU-baseline leg are the only callers.  It shares no code,
 * header, table or helper with the CUDA library, and the CUDA library never
 * calls it.
 *
 * Source of every formula: "Resumen Técnico: Atención Lineal de Orden Superior
 * (HLA)" (gist.science, paper 2510.27258).
 *   - Metodología 1 (HLA de Segundo Orden): prefix state S^K_t = sum k k^T,
 *     C^QV_t = sum q v^T, m^Q_t = sum q; cross summaries G_t, h_t; output
 *     o_t = q_t^T (S^K_t C^QV_t - G_t); ratio-normalised variant divides by the
 *     masked denominator q_t^T (S^K_t m^Q_t - h_t) (+ eps).
 *     The cross-summary updates used here are G_t = G_{t-1} + k_t k_t^T C_{t-1}
 *     and h_t = h_{t-1} + k_t k_t^T m_{t-1}, the ones the build's problem
 *     statement gives for that page.
 *   - Contribuciones 2: the masked operators "with exponential decay".  The
 *     page gives no decayed formula; the reading used is: before each token's
 *     update, every state (S, C, G, m, h) is multiplied by the head's gamma,
 *     then the undecayed updates run on the scaled values.
 *   - Contribuciones 2, the unmasked configuration: the naive product that
 *     the masked form corrects, o_t = q_t^T S^K_t C^QV_t (Metodología 1 names
 *     G_t as the correction of the future terms it includes).
 *   - Metodología 2 (AHLA): operator Q (K^T Q)(K^T V); streaming state
 *     P^KV_t = sum k v^T and E_t, with o_t = q_t^T E_t.
 *   - Metodología 2 also lists the AHLA streaming summaries (P^KV, m^K, E, n):
 *     with the value column replaced by ones, P^KV becomes m^K and E becomes n.
 *     The ratio-normalised AHLA read from that (and the ratio-normalised third
 *     order, the same way) divides the output by the same masked operator
 *     applied to a ones column, plus eps, as the second order does.
 *   - Metodología 3 (third order): A A^T A with A = Q K^T, masked, i.e.
 *     O = (M A) V with M = L (.) (A A^T), A = L (.) Q K^T; streaming with the
 *     prefix moments S^K_t, P^KV_t and the running sum F_t.
 *   - Contribuciones 2 names masked operators with exponential decay for the
 *     family, with no formula for AHLA or the third order either.  The reading
 *     is the second order's: before each token's update every state of the
 *     recurrence (AHLA: P, E; third order: S, P, F) is multiplied by gamma.
 *
 * Everything is the serial token-by-token recurrence, evaluated in double, with
 * the products written as the plain loops they are.  q_t^T (S C - G) is
 * evaluated as (q_t^T S) C - q_t^T G: the same number up to rounding order, and
 * the O(d^2 + d dv) per-token cost the page states.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* Second order (plain, ratio-normalised, decayed).                         */
/* ------------------------------------------------------------------------ */

/*
 * One head, T tokens.  q, k: [T][d]; v: [T][dv], row-major.
 * State in/out (start from zeros for a fresh sequence):
 *   S[d][d], C[d][dv], G[d][dv], m[d], h[d].
 * decay != 0: multiply all five states by gamma before every token.
 * normalized != 0: o_t = num_t / (den_t + eps), den_t = q_t^T (S m - h).
 * o: [T][dv] or NULL (state only).
 */
void oracle_hla2_head(const double* q, const double* k, const double* v,
                      int T, int d, int dv, int decay, double gamma,
                      int normalized, double eps,
                      double* S, double* C, double* G, double* m, double* h,
                      double* o)
{
    double* kC = (double*)malloc(sizeof(double) * (size_t)dv);
    double* qS = (double*)malloc(sizeof(double) * (size_t)d);
    for (int t = 0; t < T; ++t) {
        const double* qt = q + (size_t)t * d;
        const double* kt = k + (size_t)t * d;
        const double* vt = v + (size_t)t * dv;
        if (decay) {
            for (int a = 0; a < d * d; ++a) S[a] *= gamma;
            for (int a = 0; a < d * dv; ++a) { C[a] *= gamma; G[a] *= gamma; }
            for (int a = 0; a < d; ++a) { m[a] *= gamma; h[a] *= gamma; }
        }
        /* G += k (k^T C_{t-1});  h += k (k^T m_{t-1}): C, m not yet updated. */
        for (int c = 0; c < dv; ++c) {
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += kt[a] * C[(size_t)a * dv + c];
            kC[c] = s;
        }
        double km = 0.0;
        for (int a = 0; a < d; ++a) km += kt[a] * m[a];
        for (int a = 0; a < d; ++a) {
            for (int c = 0; c < dv; ++c) G[(size_t)a * dv + c] += kt[a] * kC[c];
            h[a] += kt[a] * km;
        }
        /* S += k k^T;  C += q v^T;  m += q. */
        for (int a = 0; a < d; ++a) {
            for (int b = 0; b < d; ++b) S[(size_t)a * d + b] += kt[a] * kt[b];
            for (int c = 0; c < dv; ++c) C[(size_t)a * dv + c] += qt[a] * vt[c];
            m[a] += qt[a];
        }
        if (!o) continue;
        /* o_t = q^T (S C - G) = (q^T S) C - q^T G. */
        for (int b = 0; b < d; ++b) {
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += qt[a] * S[(size_t)a * d + b];
            qS[b] = s;
        }
        double den = 0.0;
        if (normalized) {
            double sm = 0.0, qh = 0.0;
            for (int a = 0; a < d; ++a) { sm += qS[a] * m[a]; qh += qt[a] * h[a]; }
            den = sm - qh;
        }
        double* ot = o + (size_t)t * dv;
        for (int c = 0; c < dv; ++c) {
            double num = 0.0, qg = 0.0;
            for (int a = 0; a < d; ++a) {
                num += qS[a] * C[(size_t)a * dv + c];
                qg += qt[a] * G[(size_t)a * dv + c];
            }
            num -= qg;
            ot[c] = normalized ? num / (den + eps) : num;
        }
    }
    free(kC);
    free(qS);
}

/* ------------------------------------------------------------------------ */
/* Second order, unmasked inside the prefix.                                 */
/* ------------------------------------------------------------------------ */

/*
 * One head.  State in/out: S[d][d] = sum k k^T and C[d][dv] = sum q v^T, both
 * inclusive of t.  o_t = q_t^T S_t C_t, evaluated as (q_t^T S_t) C_t.
 */
void oracle_hla2u_head(const double* q, const double* k, const double* v,
                       int T, int d, int dv, double* S, double* C, double* o)
{
    double* qS = (double*)malloc(sizeof(double) * (size_t)d);
    for (int t = 0; t < T; ++t) {
        const double* qt = q + (size_t)t * d;
        const double* kt = k + (size_t)t * d;
        const double* vt = v + (size_t)t * dv;
        for (int a = 0; a < d; ++a) {
            for (int b = 0; b < d; ++b) S[(size_t)a * d + b] += kt[a] * kt[b];
            for (int c = 0; c < dv; ++c) C[(size_t)a * dv + c] += qt[a] * vt[c];
        }
        if (!o) continue;
        for (int b = 0; b < d; ++b) {
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += qt[a] * S[(size_t)a * d + b];
            qS[b] = s;
        }
        double* ot = o + (size_t)t * dv;
        for (int c = 0; c < dv; ++c) {
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += qS[a] * C[(size_t)a * dv + c];
            ot[c] = s;
        }
    }
    free(qS);
}

/* ------------------------------------------------------------------------ */
/* AHLA.                                                                     */
/* ------------------------------------------------------------------------ */

/*
 * One head.  State in/out: P[d][dv] (= sum k v^T, inclusive of t) and
 * E[d][dv] (= sum_j k_j (q_j^T P_j)).  o_t = q_t^T E_t.
 * decay != 0: P and E are multiplied by gamma before every token's update.
 */
void oracle_ahla_head(const double* q, const double* k, const double* v,
                      int T, int d, int dv, int decay, double gamma, double* P, double* E, double* o)
{
    double* qP = (double*)malloc(sizeof(double) * (size_t)dv);
    for (int t = 0; t < T; ++t) {
        const double* qt = q + (size_t)t * d;
        const double* kt = k + (size_t)t * d;
        const double* vt = v + (size_t)t * dv;
        if (decay)
            for (int a = 0; a < d * dv; ++a) { P[a] *= gamma; E[a] *= gamma; }
        for (int a = 0; a < d; ++a)
            for (int c = 0; c < dv; ++c) P[(size_t)a * dv + c] += kt[a] * vt[c];
        for (int c = 0; c < dv; ++c) {
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += qt[a] * P[(size_t)a * dv + c];
            qP[c] = s;
        }
        for (int a = 0; a < d; ++a)
            for (int c = 0; c < dv; ++c) E[(size_t)a * dv + c] += kt[a] * qP[c];
        if (!o) continue;
        double* ot = o + (size_t)t * dv;
        for (int c = 0; c < dv; ++c) {
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += qt[a] * E[(size_t)a * dv + c];
            ot[c] = s;
        }
    }
    free(qP);
}

/* ------------------------------------------------------------------------ */
/* Third order.                                                              */
/* ------------------------------------------------------------------------ */

/*
 * One head.  State in/out: S[d][d] (= sum k k^T, inclusive), P[d][dv]
 * (= sum k v^T, inclusive), F[d][dv] (= sum_s (S_s q_s)(q_s^T P_s)).
 * o_t = q_t^T F_t.  Term by term: q_t^T S_s q_s is the masked (A A^T)_{ts}
 * and q_s^T P_s is row s of A V, so o = (M A) V with M = L (.) (A A^T).
 * decay != 0: S, P and F are multiplied by gamma before every token's update.
 */
void oracle_hla3_head(const double* q, const double* k, const double* v,
                      int T, int d, int dv, int decay, double gamma, double* S, double* P, double* F, double* o)
{
    double* Sq = (double*)malloc(sizeof(double) * (size_t)d);
    double* qP = (double*)malloc(sizeof(double) * (size_t)dv);
    for (int t = 0; t < T; ++t) {
        const double* qt = q + (size_t)t * d;
        const double* kt = k + (size_t)t * d;
        const double* vt = v + (size_t)t * dv;
        if (decay) {
            for (int a = 0; a < d * d; ++a) S[a] *= gamma;
            for (int a = 0; a < d * dv; ++a) { P[a] *= gamma; F[a] *= gamma; }
        }
        for (int a = 0; a < d; ++a) {
            for (int b = 0; b < d; ++b) S[(size_t)a * d + b] += kt[a] * kt[b];
            for (int c = 0; c < dv; ++c) P[(size_t)a * dv + c] += kt[a] * vt[c];
        }
        for (int a = 0; a < d; ++a) {
            double s = 0.0;
            for (int b = 0; b < d; ++b) s += S[(size_t)a * d + b] * qt[b];
            Sq[a] = s;
        }
        for (int c = 0; c < dv; ++c) {
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += qt[a] * P[(size_t)a * dv + c];
            qP[c] = s;
        }
        for (int a = 0; a < d; ++a)
            for (int c = 0; c < dv; ++c) F[(size_t)a * dv + c] += Sq[a] * qP[c];
        if (!o) continue;
        double* ot = o + (size_t)t * dv;
        for (int c = 0; c < dv; ++c) {
            double s = 0.0;
            for (int a = 0; a < d; ++a) s += qt[a] * F[(size_t)a * dv + c];
            ot[c] = s;
        }
    }
    free(Sq);
    free(qP);
}

/* ------------------------------------------------------------------------ */
/* Many heads on host threads (full-size workloads, CPU baseline).           */
/* ------------------------------------------------------------------------ */

enum { OP_HLA2 = 0, OP_HLA2N = 1, OP_HLA2D = 2, OP_AHLA = 3, OP_HLA3 = 4, OP_HLA2U = 5, OP_AHLAN = 6,
       OP_HLA3N = 7 };


typedef struct {
    int op, BH, H, T, d, dv;
    const double *q, *k, *v, *gamma;
    double eps;
    double* o;
    int next;                /* next head to take (under lock) */
    pthread_mutex_t lock;
} job_t;

/* o = num / (den + eps), den the same operator run on a ones value column (one column). */
static void divide_by_ones_run(job_t* J, const double* q, const double* k, int T, int d, int dv, int dec, double g,
                               double* o);

static void run_head(job_t* J, int bh)
{
    const int T = J->T, d = J->d, dv = J->dv;
    const double* q = J->q + (size_t)bh * T * d;
    const double* k = J->k + (size_t)bh * T * d;
    const double* v = J->v + (size_t)bh * T * dv;
    double* o = J->o + (size_t)bh * T * dv;
    double* a = (double*)calloc((size_t)d * d, sizeof(double));
    double* b = (double*)calloc((size_t)d * dv, sizeof(double));
    double* c = (double*)calloc((size_t)d * dv, sizeof(double));
    double* m = (double*)calloc((size_t)d, sizeof(double));
    double* h = (double*)calloc((size_t)d, sizeof(double));
    /* a gamma array decays every op that has a decayed form (the unmasked one has none) */
    const int dec = J->gamma != NULL;
    const double g = dec ? J->gamma[bh % J->H] : 1.0;
    switch (J->op) {
    case OP_HLA2:
        oracle_hla2_head(q, k, v, T, d, dv, dec, g, 0, 0.0, a, b, c, m, h, o);
        break;
    case OP_HLA2N:
        oracle_hla2_head(q, k, v, T, d, dv, dec, g, 1, J->eps, a, b, c, m, h, o);
        break;
    case OP_HLA2D:
        oracle_hla2_head(q, k, v, T, d, dv, 1, g, 0, 0.0, a, b, c, m, h, o);
        break;
    case OP_AHLA:
        oracle_ahla_head(q, k, v, T, d, dv, dec, g, b, c, o);
        break;
    case OP_HLA3:
        oracle_hla3_head(q, k, v, T, d, dv, dec, g, a, b, c, o);
        break;
    case OP_HLA2U:
        oracle_hla2u_head(q, k, v, T, d, dv, a, b, o);
        break;
    case OP_AHLAN:
        oracle_ahla_head(q, k, v, T, d, dv, dec, g, b, c, o);
        divide_by_ones_run(J, q, k, T, d, dv, dec, g, o);
        break;
    case OP_HLA3N:
        oracle_hla3_head(q, k, v, T, d, dv, dec, g, a, b, c, o);
        divide_by_ones_run(J, q, k, T, d, dv, dec, g, o);
        break;
    }
    free(a); free(b); free(c); free(m); free(h);
}

static void divide_by_ones_run(job_t* J, const double* q, const double* k, int T, int d, int dv, int dec, double g,
                               double* o)
{
    double* ones = (double*)malloc(sizeof(double) * (size_t)T);
    double* den = (double*)malloc(sizeof(double) * (size_t)T);
    double* s1 = (double*)calloc((size_t)d * d, sizeof(double));
    double* s2 = (double*)calloc((size_t)d, sizeof(double));
    double* s3 = (double*)calloc((size_t)d, sizeof(double));
    for (int t = 0; t < T; ++t) ones[t] = 1.0;
    if (J->op == OP_AHLAN) oracle_ahla_head(q, k, ones, T, d, 1, dec, g, s2, s3, den);
    else oracle_hla3_head(q, k, ones, T, d, 1, dec, g, s1, s2, s3, den);
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < dv; ++c) o[(size_t)t * dv + c] /= den[t] + J->eps;
    free(ones); free(den); free(s1); free(s2); free(s3);
}

static void* worker(void* arg)
{
    job_t* J = (job_t*)arg;
    for (;;) {
        pthread_mutex_lock(&J->lock);
        int bh = J->next++;
        pthread_mutex_unlock(&J->lock);
        if (bh >= J->BH) break;
        run_head(J, bh);
    }
    return NULL;
}

/*
 * All B*H heads of one workload.  q, k: [B*H][T][d]; v, o: [B*H][T][dv];
 * gamma: [H] or NULL.  Required by OP_HLA2D; with any other op except
 * OP_HLA2U a non-NULL gamma selects that op's decayed form.  nthreads <= 0
 * means one.
 * Returns 0, or -1 on bad arguments.
 */
int oracle_forward(int op, int B, int H, int T, int d, int dv,
                   const double* q, const double* k, const double* v,
                   const double* gamma, double eps, double* o, int nthreads)
{
    if (B < 1 || H < 1 || T < 0 || d < 1 || dv < 1 || !q || !k || !v || !o) return -1;
    if (op == OP_HLA2D && !gamma) return -1;
    if (op == OP_HLA2U && gamma) return -1;
    if (op < OP_HLA2 || op > OP_HLA3N) return -1;
    job_t J;
    J.op = op; J.BH = B * H; J.H = H; J.T = T; J.d = d; J.dv = dv;
    J.q = q; J.k = k; J.v = v; J.gamma = gamma; J.eps = eps; J.o = o; J.next = 0;
    pthread_mutex_init(&J.lock, NULL);
    if (nthreads < 1) nthreads = 1;
    if (nthreads > J.BH) nthreads = J.BH;
    pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * (size_t)nthreads);
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &J);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J.lock);
    return 0;
}

/*
 * kda_oracle.c -- plain fp64 CPU oracle for Kimi Delta Attention (KDA).
 *
 * TEST INFRASTRUCTURE. Only the tests, the smoke check and the benchmark's
 * CPU-baseline leg may load or call this code; the product path (the CUDA
 * library) never does, and the two share no source, header or helper.
 *
 * What it computes, per (sequence, head), token by token, in fp64:
 *
 *   q_t <- q_t / max(||q_t||, eps),  k_t <- k_t / max(||k_t||, eps)   (if l2norm)
 *   S~  = Diag(alpha_t) S_{t-1},     alpha_t = exp(log_alpha_t)          (d_k vector)
 *   S_t = S~ + beta_t k_t (v_t - S~^T k_t)^T
 *   o_t = S_t^T q_t
 *
 * with S a d_k x d_v matrix (row = key channel, column = value channel).
 *
 * Sources (web pages, cited by title and section):
 *  - "[Kimi-2] Kimi Linear：用 KDA 重写长上下文注意力" (xutianle.me):
 *      §1, linear-attention readout o_t = S_t^T q_t;
 *      §2, delta rule as one gradient step on 1/2 ||S^T k_t - v_t||^2;
 *      §3, the boxed KDA update S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1}
 *          + beta_t k_t v_t^T and its three-step form (decay, read, correct);
 *      §5, chunkwise form: rank-1 transitions inside a chunk turned into dense
 *          products by the UT transform, output = inter-chunk state read plus
 *          intra-chunk read of earlier tokens' pseudo-values;
 *      §6.2, q and k are L2-normalised.
 *  - "Kimi Linear — 逐通道的遺忘" (docsaid.org), section "KDA：把衰減拆到每個通道":
 *      same update, S is d_k x d_v, alpha_t in [0,1]^{d_k} acts on key channels.
 *
 * Readings taken where the pages are silent: o_t reads the post-update state
 * S_t; the op itself L2-normalises q and k with eps = 1e-6 in max(||x||, eps);
 * no 1/sqrt(d) scale on q.
 *
 * Layouts (all row-major, contiguous, fp64):
 *   q, k      [T_tot][H][dk]      v, o  [T_tot][H][dv]
 *   log_alpha [T_tot][H][dk]      beta  [T_tot][H]
 *   S0, S_T   [N][H][dk][dv]      cu_seqlens [N+1] (int64, 0 = cu[0] <= ... <= cu[N] = T_tot)
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    const double *q, *k, *v, *log_alpha, *beta, *S0;
    const int64_t *cu;
    int N, H, dk, dv, l2norm, chunk;
    double eps;
    double *o, *S_T;
    int nthreads, tid;
    int status;
} job_t;

/* x / max(||x||, eps) -- the L2 normalisation of q and k (p1 §6.2). */
static void l2_normalise(const double *x, int d, int on, double eps, double *y) {
    if (!on) {
        memcpy(y, x, sizeof(double) * (size_t)d);
        return;
    }
    double ss = 0.0;
    for (int i = 0; i < d; ++i) ss += x[i] * x[i];
    double n = sqrt(ss);
    if (n < eps) n = eps;
    for (int i = 0; i < d; ++i) y[i] = x[i] / n;
}

/* One token of the KDA recurrence on state S (dk x dv), in place.
 * p1 §3: decay by Diag(alpha_t), read S~^T k_t, correct along k_t. */
static void kda_token(double *S, int dk, int dv, const double *qn, const double *kn,
                      const double *v, const double *la, double beta, double *o,
                      double *y) {
    /* S~ = Diag(alpha_t) S_{t-1}: row i (key channel i) scaled by alpha_{t,i}. */
    for (int i = 0; i < dk; ++i) {
        double a = exp(la[i]);
        double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] *= a;
    }
    /* y = S~^T k_t: what the decayed state reads at address k_t. */
    for (int j = 0; j < dv; ++j) y[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) y[j] += row[j] * kn[i];
    }
    /* S_t = S~ + k_t (beta_t (v_t - y))^T. */
    for (int j = 0; j < dv; ++j) y[j] = beta * (v[j] - y[j]);
    for (int i = 0; i < dk; ++i) {
        double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) row[j] += kn[i] * y[j];
    }
    /* o_t = S_t^T q_t. */
    for (int j = 0; j < dv; ++j) o[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) o[j] += row[j] * qn[i];
    }
}

/* Token-by-token recurrence over one (sequence, head) unit. */
static int run_recurrent_unit(const job_t *jb, int s, int h) {
    const int H = jb->H, dk = jb->dk, dv = jb->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *qn = (double *)malloc(sizeof(double) * (size_t)dk);
    double *kn = (double *)malloc(sizeof(double) * (size_t)dk);
    double *y = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!S || !qn || !kn || !y) {
        free(S); free(qn); free(kn); free(y);
        return 1;
    }
    const size_t sh = ((size_t)s * H + h) * (size_t)dk * dv;
    if (jb->S0) memcpy(S, jb->S0 + sh, sizeof(double) * (size_t)dk * dv);
    else memset(S, 0, sizeof(double) * (size_t)dk * dv);
    for (int64_t t = jb->cu[s]; t < jb->cu[s + 1]; ++t) {
        const size_t th = (size_t)t * H + h;
        l2_normalise(jb->q + th * dk, dk, jb->l2norm, jb->eps, qn);
        l2_normalise(jb->k + th * dk, dk, jb->l2norm, jb->eps, kn);
        kda_token(S, dk, dv, qn, kn, jb->v + th * dv, jb->log_alpha + th * dk,
                  jb->beta[th], jb->o + th * dv, y);
    }
    if (jb->S_T) memcpy(jb->S_T + sh, S, sizeof(double) * (size_t)dk * dv);
    free(S); free(qn); free(kn); free(y);
    return 0;
}

/*
 * Chunkwise form over one (sequence, head) unit (p1 §5, derived here).
 * Per chunk of n <= C rows with entry state S and G = inclusive cumulative
 * sum of log_alpha over the chunk's rows (per key channel):
 *   A[r][i] = sum_c k_rc k_ic exp(G_rc - G_ic)            (i <  r)
 *   P[r][i] = sum_c q_rc k_ic exp(G_rc - G_ic)            (i <= r)
 *   [W | Ut] = (I + Diag(beta) A)^-1 Diag(beta) [K*exp(G) | V]   (UT transform)
 *   U  = Ut - W S                         (pseudo-values)
 *   O  = (Q*exp(G)) S + P U               (inter-chunk + intra-chunk read)
 *   S' = Diag(exp(G_last)) S + (K*exp(G_last - G))^T U
 * It follows from unrolling S_r = Diag(alpha_r) S_{r-1} + k_r u_r^T inside the
 * chunk. Exponents are taken element-wise (exp(G_r - G_i) <= 1), never split.
 */
static int run_chunkwise_unit(const job_t *jb, int s, int h) {
    const int H = jb->H, dk = jb->dk, dv = jb->dv, C = jb->chunk;
    const size_t szS = (size_t)dk * dv;
    double *S = (double *)malloc(sizeof(double) * szS);
    double *Kc = (double *)malloc(sizeof(double) * (size_t)C * dk);
    double *Qc = (double *)malloc(sizeof(double) * (size_t)C * dk);
    double *G = (double *)malloc(sizeof(double) * (size_t)C * dk);
    double *A = (double *)malloc(sizeof(double) * (size_t)C * C);
    double *P = (double *)malloc(sizeof(double) * (size_t)C * C);
    double *X = (double *)malloc(sizeof(double) * (size_t)C * (dk + dv)); /* [W | Ut] */
    double *U = (double *)malloc(sizeof(double) * (size_t)C * dv);
    double *Snew = (double *)malloc(sizeof(double) * szS);
    if (!S || !Kc || !Qc || !G || !A || !P || !X || !U || !Snew) {
        free(S); free(Kc); free(Qc); free(G); free(A); free(P); free(X); free(U); free(Snew);
        return 1;
    }
    const size_t sh = ((size_t)s * H + h) * szS;
    if (jb->S0) memcpy(S, jb->S0 + sh, sizeof(double) * szS);
    else memset(S, 0, sizeof(double) * szS);

    for (int64_t c0 = jb->cu[s]; c0 < jb->cu[s + 1]; c0 += C) {
        int n = (int)((jb->cu[s + 1] - c0) < C ? (jb->cu[s + 1] - c0) : C);
        /* Normalised rows and cumulative log-decay G. */
        for (int r = 0; r < n; ++r) {
            const size_t th = (size_t)(c0 + r) * H + h;
            l2_normalise(jb->q + th * dk, dk, jb->l2norm, jb->eps, Qc + (size_t)r * dk);
            l2_normalise(jb->k + th * dk, dk, jb->l2norm, jb->eps, Kc + (size_t)r * dk);
            for (int c = 0; c < dk; ++c)
                G[(size_t)r * dk + c] = jb->log_alpha[th * dk + c] + (r ? G[(size_t)(r - 1) * dk + c] : 0.0);
        }
        /* A (strictly lower) and P (lower, diagonal included). */
        for (int r = 0; r < n; ++r)
            for (int i = 0; i < n; ++i) {
                double a = 0.0, p = 0.0;
                if (i <= r)
                    for (int c = 0; c < dk; ++c) {
                        double e = exp(G[(size_t)r * dk + c] - G[(size_t)i * dk + c]);
                        a += Kc[(size_t)r * dk + c] * Kc[(size_t)i * dk + c] * e;
                        p += Qc[(size_t)r * dk + c] * Kc[(size_t)i * dk + c] * e;
                    }
                A[(size_t)r * C + i] = (i < r) ? a : 0.0;
                P[(size_t)r * C + i] = (i <= r) ? p : 0.0;
            }
        /* UT transform by forward substitution:
         * X_r = beta_r (B_r - sum_{i<r} A[r][i] X_i), B_r = [k_r*exp(G_r) | v_r]. */
        const int wx = dk + dv;
        for (int r = 0; r < n; ++r) {
            const size_t th = (size_t)(c0 + r) * H + h;
            const double b = jb->beta[th];
            double *xr = X + (size_t)r * wx;
            for (int c = 0; c < dk; ++c) xr[c] = Kc[(size_t)r * dk + c] * exp(G[(size_t)r * dk + c]);
            for (int j = 0; j < dv; ++j) xr[dk + j] = jb->v[th * dv + j];
            for (int i = 0; i < r; ++i) {
                const double a = A[(size_t)r * C + i];
                const double *xi = X + (size_t)i * wx;
                for (int c = 0; c < wx; ++c) xr[c] -= a * xi[c];
            }
            for (int c = 0; c < wx; ++c) xr[c] *= b;
        }
        /* U = Ut - W S. */
        for (int r = 0; r < n; ++r) {
            const double *xr = X + (size_t)r * wx;
            for (int j = 0; j < dv; ++j) {
                double acc = xr[dk + j];
                for (int c = 0; c < dk; ++c) acc -= xr[c] * S[(size_t)c * dv + j];
                U[(size_t)r * dv + j] = acc;
            }
        }
        /* O = (Q*exp(G)) S + P U. */
        for (int r = 0; r < n; ++r) {
            const size_t th = (size_t)(c0 + r) * H + h;
            for (int j = 0; j < dv; ++j) {
                double acc = 0.0;
                for (int c = 0; c < dk; ++c)
                    acc += Qc[(size_t)r * dk + c] * exp(G[(size_t)r * dk + c]) * S[(size_t)c * dv + j];
                for (int i = 0; i <= r; ++i) acc += P[(size_t)r * C + i] * U[(size_t)i * dv + j];
                jb->o[th * dv + j] = acc;
            }
        }
        /* S' = Diag(exp(G_last)) S + (K*exp(G_last - G))^T U. */
        const double *gl = G + (size_t)(n - 1) * dk;
        for (int c = 0; c < dk; ++c)
            for (int j = 0; j < dv; ++j) {
                double acc = exp(gl[c]) * S[(size_t)c * dv + j];
                for (int r = 0; r < n; ++r)
                    acc += Kc[(size_t)r * dk + c] * exp(gl[c] - G[(size_t)r * dk + c]) * U[(size_t)r * dv + j];
                Snew[(size_t)c * dv + j] = acc;
            }
        memcpy(S, Snew, sizeof(double) * szS);
    }
    if (jb->S_T) memcpy(jb->S_T + sh, S, sizeof(double) * szS);
    free(S); free(Kc); free(Qc); free(G); free(A); free(P); free(X); free(U); free(Snew);
    return 0;
}

/* Units (sequence, head) are independent; thread `tid` takes every nthreads-th one. */
static void *worker(void *arg) {
    job_t *jb = (job_t *)arg;
    const int units = jb->N * jb->H;
    for (int u = jb->tid; u < units; u += jb->nthreads) {
        int s = u / jb->H, h = u % jb->H;
        int rc = jb->chunk > 0 ? run_chunkwise_unit(jb, s, h) : run_recurrent_unit(jb, s, h);
        if (rc) jb->status = rc;
    }
    return NULL;
}

static int run_all(job_t base) {
    int nt = base.nthreads < 1 ? 1 : base.nthreads;
    if (nt > base.N * base.H) nt = base.N * base.H;
    if (nt < 1) nt = 1;
    job_t *jobs = (job_t *)calloc((size_t)nt, sizeof(job_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nt, sizeof(pthread_t));
    if (!jobs || !th) { free(jobs); free(th); return 1; }
    for (int i = 0; i < nt; ++i) {
        jobs[i] = base;
        jobs[i].nthreads = nt;
        jobs[i].tid = i;
        jobs[i].status = 0;
    }
    for (int i = 1; i < nt; ++i)
        if (pthread_create(&th[i], NULL, worker, &jobs[i])) jobs[i].status = 2;
    worker(&jobs[0]);
    int status = jobs[0].status;
    for (int i = 1; i < nt; ++i) {
        if (jobs[i].status != 2) pthread_join(th[i], NULL);
        if (jobs[i].status) status = jobs[i].status;
    }
    free(jobs); free(th);
    return status;
}

static int check_args(const int64_t *cu, int N, int H, int dk, int dv) {
    if (!cu || N < 1 || H < 1 || dk < 1 || dv < 1) return 3;
    if (cu[0] != 0) return 3;
    for (int s = 0; s < N; ++s) if (cu[s + 1] < cu[s]) return 3;
    return 0;
}

/* Token-by-token recurrence (the definition). Returns 0 on success. */
int kda_oracle_recurrent(const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *S0,
                         const int64_t *cu_seqlens, int N, int H, int dk, int dv,
                         int l2norm, double eps, double *o, double *S_T, int nthreads) {
    int rc = check_args(cu_seqlens, N, H, dk, dv);
    if (rc) return rc;
    job_t jb = {q, k, v, log_alpha, beta, S0, cu_seqlens, N, H, dk, dv, l2norm, 0,
                eps, o, S_T, nthreads, 0, 0};
    return run_all(jb);
}

/* Chunkwise form with chunk size `chunk` >= 1 (same outputs up to rounding). */
int kda_oracle_chunkwise(const double *q, const double *k, const double *v,
                         const double *log_alpha, const double *beta, const double *S0,
                         const int64_t *cu_seqlens, int N, int H, int dk, int dv,
                         int l2norm, double eps, int chunk, double *o, double *S_T,
                         int nthreads) {
    int rc = check_args(cu_seqlens, N, H, dk, dv);
    if (rc) return rc;
    if (chunk < 1) return 3;
    job_t jb = {q, k, v, log_alpha, beta, S0, cu_seqlens, N, H, dk, dv, l2norm, chunk,
                eps, o, S_T, nthreads, 0, 0};
    return run_all(jb);
}

/* One decode step: N sequences x H heads, one token each, state S updated in
 * place ([N][H][dk][dv]); inputs are [N][H][d]. The recurrence for one token. */
int kda_oracle_decode_step(const double *q, const double *k, const double *v,
                           const double *log_alpha, const double *beta, double *S,
                           int N, int H, int dk, int dv, int l2norm, double eps,
                           double *o) {
    if (N < 1 || H < 1 || dk < 1 || dv < 1) return 3;
    double *qn = (double *)malloc(sizeof(double) * (size_t)dk);
    double *kn = (double *)malloc(sizeof(double) * (size_t)dk);
    double *y = (double *)malloc(sizeof(double) * (size_t)dv);
    if (!qn || !kn || !y) { free(qn); free(kn); free(y); return 1; }
    for (int s = 0; s < N; ++s)
        for (int h = 0; h < H; ++h) {
            const size_t th = (size_t)s * H + h;
            l2_normalise(q + th * dk, dk, l2norm, eps, qn);
            l2_normalise(k + th * dk, dk, l2norm, eps, kn);
            kda_token(S + th * (size_t)dk * dv, dk, dv, qn, kn, v + th * dv,
                      log_alpha + th * dk, beta[th], o + th * dv, y);
        }
    free(qn); free(kn); free(y);
    return 0;
}

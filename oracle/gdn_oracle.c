/*
 * gdn_oracle.c -- plain, slow, fp64 CPU oracle for the Gated DeltaNet
 * token-mixer recurrence.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header or constant with the CUDA
 * library.
 *
 * What it computes (the plain definition, token by token, in double):
 *
 *   Qwen3.8-Flash-Next summary (picx.dev), "Theoretical foundations",
 *   eqs. (1)-(4), per head with S in R^{dk x dv}:
 *       St  = alpha_t * S_{t-1}                      (1)
 *       e_t = v_t - St^T k_t                         (2)
 *       S_t = St + beta_t * k_t e_t^T                (3)
 *       y_t = S_t^T q_t                              (4)
 *   with alpha_t, beta_t in (0,1) scalars per token and head (same passage).
 *
 *   Same page, "Methodology" / "1. GDN Hybrid Token Mixing": q and k are L2
 *   normalised.  The pages give no formula; the reading used here is
 *   x_hat = x / sqrt(sum(x^2) + eps), switchable off (l2norm = 0).
 *
 *   y is multiplied by `scale` (1 by default; eq. (4) has none).
 *
 * The backward pass is the reverse-mode derivative of exactly these steps,
 * taken one token at a time in reverse order (chain rule, written out in
 * chain_backward below).  States S_{t-1} are kept every SEG tokens and the
 * forward recurrence is replayed inside each segment.
 *
 * Layouts (row-major, last index fastest), all double:
 *   dense : q,k [B,T,H,dk]  v,y,dy [B,T,H,dv]  alpha,beta [B,T,H]
 *           S0, S_final, dS0, dS_final [B,H,dk,dv]
 *   varlen: tokens packed as [1,Ttot,H,*]; document n covers tokens
 *           cu[n] .. cu[n+1]-1; states are [N,H,dk,dv].
 * Each (sequence, head) pair is an independent chain; chains are spread over
 * threads, the loop inside a chain is sequential.
 *
 * Return value of every entry point: 0 on success, -1 on a bad argument,
 * -2 when memory could not be allocated.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define SEG 64 /* tokens between stored states in the backward pass */

/* A chain: token indices t0..t1-1 of the packed [Ttot, H, *] arrays, head h,
 * state slot `slot` of the [*, H, dk, dv] state arrays. */
typedef struct {
    long t0, t1;
    int h, slot;
} chain_t;

typedef struct {
    /* inputs */
    const double *q, *k, *v, *alpha, *beta, *s0, *dy, *ds_final;
    /* outputs */
    double *y, *s_final, *dq, *dk, *dv, *dalpha, *dbeta, *ds0;
    int H, DK, DV;
    double scale, eps;
    int l2norm;
    const chain_t* chains;
    long nchains;
    long next; /* work counter, guarded by mu */
    pthread_mutex_t mu;
    int failed;
} job_t;

/* ---------------------------------------------------------------- helpers */

/* x_hat = x / sqrt(|x|^2 + eps); also returns 1/sqrt(|x|^2 + eps). */
static double l2norm_vec(const double* x, int n, double eps, int on, double* out) {
    if (!on) {
        for (int i = 0; i < n; ++i) out[i] = x[i];
        return 1.0;
    }
    double ss = 0.0;
    for (int i = 0; i < n; ++i) ss += x[i] * x[i];
    double r = 1.0 / sqrt(ss + eps);
    for (int i = 0; i < n; ++i) out[i] = x[i] * r;
    return r;
}

/* Gradient through the normalisation:
 * dx = (dxh - xh * <xh, dxh>) * r  where r = 1/sqrt(|x|^2+eps). */
static void l2norm_vec_backward(const double* xh, const double* dxh, double r, int n, int on,
                                double* dx) {
    if (!on) {
        for (int i = 0; i < n; ++i) dx[i] = dxh[i];
        return;
    }
    double dot = 0.0;
    for (int i = 0; i < n; ++i) dot += xh[i] * dxh[i];
    for (int i = 0; i < n; ++i) dx[i] = (dxh[i] - xh[i] * dot) * r;
}

/* One token of eqs. (1)-(4) in place on S (dk x dv, row-major).
 * kh, qh are the normalised key and query; e (dv) receives the error. */
static void gdn_step(double* S, const double* kh, const double* qh, const double* v, double a,
                     double b, double scale, double* y, double* e, int DK, int DV) {
    /* (1) St = a * S */
    for (int i = 0; i < DK * DV; ++i) S[i] *= a;
    /* (2) e = v - St^T kh */
    for (int j = 0; j < DV; ++j) {
        double p = 0.0;
        for (int i = 0; i < DK; ++i) p += S[i * DV + j] * kh[i];
        e[j] = v[j] - p;
    }
    /* (3) S = St + b * kh e^T */
    for (int i = 0; i < DK; ++i)
        for (int j = 0; j < DV; ++j) S[i * DV + j] += b * kh[i] * e[j];
    /* (4) y = scale * S^T qh */
    if (y) {
        for (int j = 0; j < DV; ++j) {
            double acc = 0.0;
            for (int i = 0; i < DK; ++i) acc += S[i * DV + j] * qh[i];
            y[j] = scale * acc;
        }
    }
}

/* ----------------------------------------------------------------- forward */

static void chain_forward(job_t* J, const chain_t* c, double* S, double* kh, double* qh,
                          double* e) {
    const int H = J->H, DK = J->DK, DV = J->DV;
    const size_t ssz = (size_t)DK * DV;
    const size_t soff = ((size_t)c->slot * H + c->h) * ssz;
    if (J->s0)
        memcpy(S, J->s0 + soff, ssz * sizeof(double));
    else
        memset(S, 0, ssz * sizeof(double));
    for (long t = c->t0; t < c->t1; ++t) {
        const size_t th = (size_t)t * H + c->h;
        l2norm_vec(J->k + th * DK, DK, J->eps, J->l2norm, kh);
        l2norm_vec(J->q + th * DK, DK, J->eps, J->l2norm, qh);
        gdn_step(S, kh, qh, J->v + th * DV, J->alpha[th], J->beta[th], J->scale,
                 J->y ? J->y + th * DV : NULL, e, DK, DV);
    }
    if (J->s_final) memcpy(J->s_final + soff, S, ssz * sizeof(double));
}

/* ---------------------------------------------------------------- backward */

/*
 * Reverse mode through one chain.  For t = t1-1 down to t0, with dS holding
 * dL/dS_t (initialised from dS_final):
 *   y_t = scale S_t^T qh          => dS += scale qh dy^T ;  dqh = scale S_t dy
 *   S_t = St + b kh e^T           => dSt = dS ; db = kh^T dS e ;
 *                                    dkh = b dS e ;  de = b dS^T kh
 *   e   = v - St^T kh             => dv = de ; dSt -= kh de^T ; dkh -= St de
 *   St  = a S_{t-1}               => da = <dSt, S_{t-1}> ; dS_{t-1} = a dSt
 * and finally dS0 = dS.  dq, dk go back through the normalisation.
 */
static int chain_backward(job_t* J, const chain_t* c) {
    const int H = J->H, DK = J->DK, DV = J->DV;
    const size_t ssz = (size_t)DK * DV;
    const size_t soff = ((size_t)c->slot * H + c->h) * ssz;
    const long L = c->t1 - c->t0;
    const long nseg = (L + SEG - 1) / SEG;

    double* seg_start = malloc((size_t)(nseg > 0 ? nseg : 1) * ssz * sizeof(double));
    double* states = malloc((size_t)(SEG + 1) * ssz * sizeof(double)); /* S before/after */
    double* dS = malloc(ssz * sizeof(double));
    double* dSt = malloc(ssz * sizeof(double));
    double* St = malloc(ssz * sizeof(double));
    double* wk = malloc((size_t)(6 * DK + 3 * DV) * sizeof(double));
    if (!seg_start || !states || !dS || !dSt || !St || !wk) {
        free(seg_start); free(states); free(dS); free(dSt); free(St); free(wk);
        return -2;
    }
    double *kh = wk, *qh = wk + DK, *dkh = wk + 2 * DK, *dqh = wk + 3 * DK;
    double *dxk = wk + 4 * DK, *dxq = wk + 5 * DK;
    double *e = wk + 6 * DK, *de = e + DV, *dyv = de + DV;

    /* forward pass storing the state at the start of every segment */
    double* S = states;
    if (J->s0)
        memcpy(S, J->s0 + soff, ssz * sizeof(double));
    else
        memset(S, 0, ssz * sizeof(double));
    for (long t = c->t0; t < c->t1; ++t) {
        if ((t - c->t0) % SEG == 0) memcpy(seg_start + ((t - c->t0) / SEG) * ssz, S, ssz * sizeof(double));
        const size_t th = (size_t)t * H + c->h;
        l2norm_vec(J->k + th * DK, DK, J->eps, J->l2norm, kh);
        l2norm_vec(J->q + th * DK, DK, J->eps, J->l2norm, qh);
        gdn_step(S, kh, qh, J->v + th * DV, J->alpha[th], J->beta[th], J->scale, NULL, e, DK, DV);
    }

    if (J->ds_final)
        memcpy(dS, J->ds_final + soff, ssz * sizeof(double));
    else
        memset(dS, 0, ssz * sizeof(double));

    for (long sgi = nseg - 1; sgi >= 0; --sgi) {
        const long a0 = c->t0 + sgi * SEG;
        const long a1 = (a0 + SEG < c->t1) ? a0 + SEG : c->t1;
        /* replay: states[i] = S before token a0+i; states[n] = S after the last */
        memcpy(states, seg_start + sgi * ssz, ssz * sizeof(double));
        for (long t = a0; t < a1; ++t) {
            const size_t th = (size_t)t * H + c->h;
            double* Sn = states + (size_t)(t - a0 + 1) * ssz;
            memcpy(Sn, states + (size_t)(t - a0) * ssz, ssz * sizeof(double));
            l2norm_vec(J->k + th * DK, DK, J->eps, J->l2norm, kh);
            l2norm_vec(J->q + th * DK, DK, J->eps, J->l2norm, qh);
            gdn_step(Sn, kh, qh, J->v + th * DV, J->alpha[th], J->beta[th], J->scale, NULL, e, DK,
                     DV);
        }
        for (long t = a1 - 1; t >= a0; --t) {
            const size_t th = (size_t)t * H + c->h;
            const double* Sprev = states + (size_t)(t - a0) * ssz;
            const double* Scur = states + (size_t)(t - a0 + 1) * ssz;
            const double a = J->alpha[th], b = J->beta[th];
            const double rk = l2norm_vec(J->k + th * DK, DK, J->eps, J->l2norm, kh);
            const double rq = l2norm_vec(J->q + th * DK, DK, J->eps, J->l2norm, qh);
            const double* vv = J->v + th * DV;
            for (int j = 0; j < DV; ++j) dyv[j] = J->dy ? J->dy[th * DV + j] : 0.0;

            /* St = a * S_{t-1};  e = v - St^T kh */
            for (size_t i = 0; i < ssz; ++i) St[i] = a * Sprev[i];
            for (int j = 0; j < DV; ++j) {
                double p = 0.0;
                for (int i = 0; i < DK; ++i) p += St[i * DV + j] * kh[i];
                e[j] = vv[j] - p;
            }
            /* output: dS += scale qh dy^T ; dqh = scale S_t dy */
            for (int i = 0; i < DK; ++i) {
                double acc = 0.0;
                for (int j = 0; j < DV; ++j) {
                    dS[i * DV + j] += J->scale * qh[i] * dyv[j];
                    acc += Scur[i * DV + j] * dyv[j];
                }
                dqh[i] = J->scale * acc;
            }
            /* update: db, dkh (first part), de */
            double db = 0.0;
            for (int i = 0; i < DK; ++i) {
                double acc = 0.0;
                for (int j = 0; j < DV; ++j) acc += dS[i * DV + j] * e[j];
                db += kh[i] * acc;
                dkh[i] = b * acc;
            }
            for (int j = 0; j < DV; ++j) {
                double acc = 0.0;
                for (int i = 0; i < DK; ++i) acc += dS[i * DV + j] * kh[i];
                de[j] = b * acc;
            }
            /* error: dv = de ; dSt = dS - kh de^T ; dkh -= St de */
            for (int i = 0; i < DK; ++i) {
                double acc = 0.0;
                for (int j = 0; j < DV; ++j) {
                    dSt[i * DV + j] = dS[i * DV + j] - kh[i] * de[j];
                    acc += St[i * DV + j] * de[j];
                }
                dkh[i] -= acc;
            }
            /* decay: da = <dSt, S_{t-1}> ; dS_{t-1} = a dSt */
            double da = 0.0;
            for (size_t i = 0; i < ssz; ++i) da += dSt[i] * Sprev[i];
            for (size_t i = 0; i < ssz; ++i) dS[i] = a * dSt[i];

            l2norm_vec_backward(kh, dkh, rk, DK, J->l2norm, dxk);
            l2norm_vec_backward(qh, dqh, rq, DK, J->l2norm, dxq);
            for (int i = 0; i < DK; ++i) {
                J->dk[th * DK + i] = dxk[i];
                J->dq[th * DK + i] = dxq[i];
            }
            for (int j = 0; j < DV; ++j) J->dv[th * DV + j] = de[j];
            J->dalpha[th] = da;
            J->dbeta[th] = db;
        }
    }
    if (J->ds0) memcpy(J->ds0 + soff, dS, ssz * sizeof(double));

    free(seg_start); free(states); free(dS); free(dSt); free(St); free(wk);
    return 0;
}

/* ------------------------------------------------------------- threading */

typedef struct {
    job_t* J;
    int backward;
} worker_arg_t;

static void* worker(void* p) {
    worker_arg_t* w = (worker_arg_t*)p;
    job_t* J = w->J;
    const int DK = J->DK, DV = J->DV;
    double* S = malloc((size_t)DK * DV * sizeof(double));
    double* buf = malloc((size_t)(2 * DK + DV) * sizeof(double));
    if (!S || !buf) {
        pthread_mutex_lock(&J->mu);
        J->failed = 1;
        pthread_mutex_unlock(&J->mu);
        free(S); free(buf);
        return NULL;
    }
    for (;;) {
        pthread_mutex_lock(&J->mu);
        long i = J->next++;
        pthread_mutex_unlock(&J->mu);
        if (i >= J->nchains) break;
        if (w->backward) {
            if (chain_backward(J, &J->chains[i]) != 0) {
                pthread_mutex_lock(&J->mu);
                J->failed = 1;
                pthread_mutex_unlock(&J->mu);
            }
        } else {
            chain_forward(J, &J->chains[i], S, buf, buf + DK, buf + 2 * DK);
        }
    }
    free(S); free(buf);
    return NULL;
}

static int run_job(job_t* J, int nthreads, int backward) {
    if (nthreads <= 0) {
        long n = sysconf(_SC_NPROCESSORS_ONLN);
        nthreads = n > 0 ? (int)n : 1;
    }
    if (nthreads > J->nchains) nthreads = (int)(J->nchains > 0 ? J->nchains : 1);
    J->next = 0;
    J->failed = 0;
    pthread_mutex_init(&J->mu, NULL);
    pthread_t* th = malloc((size_t)nthreads * sizeof(pthread_t));
    worker_arg_t w = {J, backward};
    if (!th) return -2;
    int started = 0;
    for (int i = 0; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, worker, &w) == 0) ++started;
        else break;
    }
    if (started == 0) worker(&w);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    pthread_mutex_destroy(&J->mu);
    return J->failed ? -2 : 0;
}

static chain_t* dense_chains(int B, int T, int H) {
    chain_t* c = malloc((size_t)B * H * sizeof(chain_t));
    if (!c) return NULL;
    for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h) {
            chain_t* x = &c[(size_t)b * H + h];
            x->t0 = (long)b * T;
            x->t1 = (long)b * T + T;
            x->h = h;
            x->slot = b;
        }
    return c;
}

static chain_t* varlen_chains(const int* cu, int N, int H) {
    chain_t* c = malloc((size_t)N * H * sizeof(chain_t));
    if (!c) return NULL;
    for (int n = 0; n < N; ++n)
        for (int h = 0; h < H; ++h) {
            chain_t* x = &c[(size_t)n * H + h];
            x->t0 = cu[n];
            x->t1 = cu[n + 1];
            x->h = h;
            x->slot = n;
        }
    return c;
}

/* ------------------------------------------------------------ entry points */

int gdn_oracle_forward(const double* q, const double* k, const double* v, const double* alpha,
                       const double* beta, const double* s0, double* y, double* s_final, int B,
                       int T, int H, int dk, int dv, double scale, int l2norm, double eps,
                       int nthreads) {
    if (!q || !k || !v || !alpha || !beta || B < 0 || T < 0 || H < 1 || dk < 1 || dv < 1)
        return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.s0 = s0;
    J.y = y; J.s_final = s_final;
    J.H = H; J.DK = dk; J.DV = dv; J.scale = scale; J.eps = eps; J.l2norm = l2norm;
    chain_t* c = dense_chains(B, T, H);
    if (!c && B > 0) return -2;
    J.chains = c;
    J.nchains = (long)B * H;
    int rc = run_job(&J, nthreads, 0);
    free(c);
    return rc;
}

int gdn_oracle_forward_varlen(const double* q, const double* k, const double* v,
                              const double* alpha, const double* beta, const int* cu_seqlens,
                              int num_seqs, const double* s0, double* y, double* s_final,
                              int H, int dk, int dv, double scale, int l2norm, double eps,
                              int nthreads) {
    if (!cu_seqlens || num_seqs < 0 || H < 1 || dk < 1 || dv < 1) return -1;
    if (num_seqs > 0 && cu_seqlens[0] != 0) return -1;
    for (int n = 0; n < num_seqs; ++n)
        if (cu_seqlens[n + 1] < cu_seqlens[n]) return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.s0 = s0;
    J.y = y; J.s_final = s_final;
    J.H = H; J.DK = dk; J.DV = dv; J.scale = scale; J.eps = eps; J.l2norm = l2norm;
    chain_t* c = varlen_chains(cu_seqlens, num_seqs, H);
    if (!c && num_seqs > 0) return -2;
    J.chains = c;
    J.nchains = (long)num_seqs * H;
    int rc = run_job(&J, nthreads, 0);
    free(c);
    return rc;
}

int gdn_oracle_backward(const double* q, const double* k, const double* v, const double* alpha,
                        const double* beta, const double* s0, const double* dy,
                        const double* ds_final, double* dq, double* dk_out, double* dv_out,
                        double* dalpha, double* dbeta, double* ds0, int B, int T, int H, int dk,
                        int dv, double scale, int l2norm, double eps, int nthreads) {
    if (!q || !k || !v || !alpha || !beta || !dq || !dk_out || !dv_out || !dalpha || !dbeta ||
        B < 0 || T < 0 || H < 1 || dk < 1 || dv < 1)
        return -1;
    job_t J;
    memset(&J, 0, sizeof(J));
    J.q = q; J.k = k; J.v = v; J.alpha = alpha; J.beta = beta; J.s0 = s0;
    J.dy = dy; J.ds_final = ds_final;
    J.dq = dq; J.dk = dk_out; J.dv = dv_out; J.dalpha = dalpha; J.dbeta = dbeta; J.ds0 = ds0;
    J.H = H; J.DK = dk; J.DV = dv; J.scale = scale; J.eps = eps; J.l2norm = l2norm;
    chain_t* c = dense_chains(B, T, H);
    if (!c && B > 0) return -2;
    J.chains = c;
    J.nchains = (long)B * H;
    int rc = run_job(&J, nthreads, 1);
    free(c);
    return rc;
}

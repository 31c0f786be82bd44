/*
 * KDA oracle: a plain, slow, fp64 CPU implementation of one KDA sequence-mixing
 * step, used only as test infrastructure (parity tests, the smoke check and the
 * CPU baseline leg of the benchmark).  Nothing on the product path may call it.
 *
 * Definition followed ("GLM-5.3-Flash im Detail", section "Sequenz-Mixing:
 * 34 KDA-Schichten mit festem Zustand"): query, key and value each pass a causal
 * depthwise convolution of width four; a per-channel forget gate decays the
 * state; a scalar beta controls a delta-rule write; the query reads the updated
 * state; 64 heads of dimension 128; the log-decay is bounded below by -5.
 * The same section says prefill evaluates tokens chunk-parallel while decode does
 * one recurrent update per token.  The exact recurrence written out below is
 *
 *     S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T
 *     o_t = S_t^T q_t
 *
 * with alpha_t = exp(max(g_t, -5)) per key channel, S a d_k x d_v matrix (row =
 * key channel, column = value channel) and q_t, k_t the conv outputs divided by
 * sqrt(||.||^2 + 1e-6).  This file evaluates it token by token in the expanded
 * form  S <- Diag(alpha) S;  r = S^T k;  S <- S + beta k (v - r)^T;  o = S^T q,
 * which is the product above multiplied out (no reordering across tokens).
 *
 * Readings where the pages are silent (each one is listed in the design notes):
 *   - conv tap j in 0..3 multiplies token t-3+j (tap 3 = current token), no bias,
 *     tokens before the segment come from init_conv (zeros when NULL);
 *   - conv activation: none by default, SiLU (y * sigmoid(y)) when act == 1;
 *   - L2 norm epsilon 1e-6 inside the square root; v is not normalised;
 *   - the lower bound is applied as g' = max(g, -5); no query scale.
 *
 * Everything here is fp64.  Inputs are taken as the exact values of their stored
 * (bf16 / fp32) representation, converted to double by the caller.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define KDA_ORACLE_LOG_DECAY_FLOOR (-5.0)
#define KDA_ORACLE_NORM_EPS (1e-6)

typedef struct {
    int64_t T;              /* tokens in this segment (may be 0)                   */
    int dk, dv;             /* key / value head dims                               */
    const double *q, *k;    /* [T][dk] raw (pre-conv) queries / keys               */
    const double *v;        /* [T][dv] raw values                                  */
    const double *g;        /* [T][dk] log-decay (before the -5 floor)             */
    const double *beta;     /* [T]                                                 */
    const double *wq, *wk;  /* [dk][4] conv taps for this head                     */
    const double *wv;       /* [dv][4]                                             */
    const double *init_state; /* [dk][dv] or NULL (zero)                           */
    const double *cq, *ck;  /* [3][dk] conv history, oldest first, or NULL (zero)  */
    const double *cv;       /* [3][dv]                                             */
    int act;                /* 0 = none, 1 = SiLU                                  */
    double *o;              /* [T][dv] out                                         */
    double *final_state;    /* [dk][dv] out                                        */
    double *tq, *tk;        /* [3][dk] out: last 3 raw tokens of history+segment   */
    double *tv;             /* [3][dv] out                                         */
    int state_round;        /* state storage: 0 = kept exact; 1 = rounded to bf16  */
                            /* after every token (each token is one decode step    */
                            /* whose state is stored); 2 = rounded to bf16 once,   */
                            /* when the final state is stored                      */
} kda_oracle_job;

/* Round x to the nearest bfloat16 value (8 significant bits, exponent range
 * of fp32), ties to even, directly from double (no intermediate float, so no
 * double rounding).  |x| is far below the bf16 overflow threshold for states;
 * larger values are not handled. */
static double round_bf16(double x) {
    if (x == 0.0 || !isfinite(x)) return x;
    int e;
    frexp(x, &e);                 /* |x| = m 2^e, 0.5 <= m < 1                   */
    int shift = 8 - e;            /* 8 significant bits: ulp = 2^(e - 8)         */
    if (e - 8 < -133) shift = 133;  /* bf16 subnormals: ulp 2^-133               */
    return ldexp(nearbyint(ldexp(x, shift)), -shift);  /* default mode: ties even */
}

/* y_t[c] = sum_j w[c][j] * x_{t-3+j}[c], x_{<0} from the 3-token history. */
static double conv_at(const double *x, const double *hist, const double *w,
                      int64_t t, int c, int d, int act) {
    double y = 0.0;
    for (int j = 0; j < 4; ++j) {
        int64_t s = t - 3 + j;
        double xs;
        if (s >= 0)
            xs = x[s * d + c];
        else
            xs = hist ? hist[(3 + s) * d + c] : 0.0;  /* s in -3..-1 -> hist row 0..2 */
        y += w[c * 4 + j] * xs;
    }
    if (act == 1) y = y / (1.0 + exp(-y));
    return y;
}

/* last three raw tokens of concat(history, segment), oldest first */
static void conv_tail(const double *x, const double *hist, int64_t T, int d, double *out) {
    for (int r = 0; r < 3; ++r) {
        int64_t s = T - 3 + r;  /* position in the segment; negative -> history */
        for (int c = 0; c < d; ++c) {
            double val;
            if (s >= 0)
                val = x[s * d + c];
            else
                val = hist ? hist[(3 + s) * d + c] : 0.0;
            out[r * d + c] = val;
        }
    }
}

void kda_oracle_run_job(const kda_oracle_job *jb) {
    const int dk = jb->dk, dv = jb->dv;
    double *S = (double *)malloc(sizeof(double) * (size_t)dk * dv);
    double *qh = (double *)malloc(sizeof(double) * dk);
    double *kh = (double *)malloc(sizeof(double) * dk);
    double *al = (double *)malloc(sizeof(double) * dk);
    double *vv = (double *)malloc(sizeof(double) * dv);
    double *r = (double *)malloc(sizeof(double) * dv);

    if (jb->init_state)
        memcpy(S, jb->init_state, sizeof(double) * (size_t)dk * dv);
    else
        memset(S, 0, sizeof(double) * (size_t)dk * dv);

    for (int64_t t = 0; t < jb->T; ++t) {
        /* 1. causal depthwise conv on q, k, v */
        double nq = 0.0, nk = 0.0;
        for (int c = 0; c < dk; ++c) {
            qh[c] = conv_at(jb->q, jb->cq, jb->wq, t, c, dk, jb->act);
            kh[c] = conv_at(jb->k, jb->ck, jb->wk, t, c, dk, jb->act);
            nq += qh[c] * qh[c];
            nk += kh[c] * kh[c];
        }
        for (int c = 0; c < dv; ++c) vv[c] = conv_at(jb->v, jb->cv, jb->wv, t, c, dv, jb->act);
        /* 2. L2 normalisation of q and k */
        nq = 1.0 / sqrt(nq + KDA_ORACLE_NORM_EPS);
        nk = 1.0 / sqrt(nk + KDA_ORACLE_NORM_EPS);
        for (int c = 0; c < dk; ++c) {
            qh[c] *= nq;
            kh[c] *= nk;
        }
        /* 3. per-channel decay with the log-decay floor */
        for (int c = 0; c < dk; ++c) {
            double gc = jb->g[t * dk + c];
            if (gc < KDA_ORACLE_LOG_DECAY_FLOOR) gc = KDA_ORACLE_LOG_DECAY_FLOOR;
            al[c] = exp(gc);
        }
        const double b = jb->beta[t];
        /* 4. S <- Diag(alpha) S */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[i * dv + j] *= al[i];
        /* r = S^T k */
        for (int j = 0; j < dv; ++j) r[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) r[j] += S[i * dv + j] * kh[i];
        /* S <- S + beta k (v - r)^T   (equals (I - beta k k^T) S + beta k v^T) */
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) S[i * dv + j] += b * kh[i] * (vv[j] - r[j]);
        /* 5. o = S^T q */
        double *ot = jb->o + t * dv;
        for (int j = 0; j < dv; ++j) ot[j] = 0.0;
        for (int i = 0; i < dk; ++i)
            for (int j = 0; j < dv; ++j) ot[j] += S[i * dv + j] * qh[i];
        /* 6. a decode step stores its state: in bf16 storage the next token
         *    starts from the stored (rounded) values; the readout above used
         *    the state before storage */
        if (jb->state_round == 1)
            for (int i = 0; i < dk * dv; ++i) S[i] = round_bf16(S[i]);
    }
    if (jb->state_round == 2)
        for (int i = 0; i < dk * dv; ++i) S[i] = round_bf16(S[i]);
    memcpy(jb->final_state, S, sizeof(double) * (size_t)dk * dv);
    conv_tail(jb->q, jb->cq, jb->T, dk, jb->tq);
    conv_tail(jb->k, jb->ck, jb->T, dk, jb->tk);
    conv_tail(jb->v, jb->cv, jb->T, dv, jb->tv);

    free(S); free(qh); free(kh); free(al); free(vv); free(r);
}

typedef struct {
    const kda_oracle_job *jobs;
    int njobs;
    int stride, first;
} worker_arg;

static void *worker(void *p) {
    worker_arg *a = (worker_arg *)p;
    for (int i = a->first; i < a->njobs; i += a->stride) kda_oracle_run_job(&a->jobs[i]);
    return NULL;
}

/* Runs independent (sequence, head) jobs on up to nthreads POSIX threads.
 * Returns the number of threads actually used. */
int kda_oracle_run_jobs(const kda_oracle_job *jobs, int njobs, int nthreads) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > njobs) nthreads = njobs;
    if (nthreads <= 1) {
        for (int i = 0; i < njobs; ++i) kda_oracle_run_job(&jobs[i]);
        return 1;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    worker_arg *args = (worker_arg *)malloc(sizeof(worker_arg) * nthreads);
    for (int t = 0; t < nthreads; ++t) {
        args[t].jobs = jobs;
        args[t].njobs = njobs;
        args[t].stride = nthreads;
        args[t].first = t;
        pthread_create(&th[t], NULL, worker, &args[t]);
    }
    for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(th);
    free(args);
    return nthreads;
}

int kda_oracle_job_size(void) { return (int)sizeof(kda_oracle_job); }

/* The bf16 rounding above, exposed for its pin tests. */
void kda_oracle_round_bf16(const double *x, double *y, int64_t n) {
    for (int64_t i = 0; i < n; ++i) y[i] = round_bf16(x[i]);
}

/*
 * la_oracle.c -- plain, slow, fp64 CPU oracle for linear attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may call, link or
 * load this file: only the tests, the smoke check and the benchmark's CPU
 * baseline / reference arm use it.  It shares no code, header, table or
 * helper with the CUDA library; it sees the same (already rounded) input
 * values, widened exactly to double.
 *
 * Sources (web pages on the subject):
 *  - "Flash Bi-directional Linear Attention" README (fla-org), intro and
 *    "Update" list: bidirectional (non-causal) linear attention `linear_attn`
 *    with a norm term, and `simple_la`, the same without the norm term.
 *  - "flash-linear-attention" README (sustcsonglin), "Benchmarks" (RetNet,
 *    i.e. retention) and "Different forms of linear attention"
 *    (Parallel / FusedRecurrent / FusedChunk / ParallelChunk).
 *
 * The pages name the operations but print no formulas; the definitions used
 * here are the plain readings (every one is listed in the design notes):
 *
 *   phi(x)  = elu(x) + 1  = x + 1 (x > 0),  exp(x) (x <= 0)
 *   bidir:   S = sum_s phi(k_s)^T v_s (D x D),  z = sum_s phi(k_s) (D)
 *            o_t = phi(q_t) S / (phi(q_t) . z + eps)
 *   simple:  o_t = q_t (sum_s k_s^T v_s)            (identity phi, no norm)
 *   retention (causal, per-head scalar decay gamma_h):
 *            o_t = sum_{s<=t} gamma^(t-s) (q_t . k_s) v_s
 *            computed in the recurrent ("FusedRecurrent") form
 *            S_t = gamma S_{t-1} + k_t^T v_t,  o_t = q_t S_t.
 *   gated (data-dependent decay per token and key dimension, g_t <= 0 the log gates):
 *            S_t = diag(exp(g_t)) S_{t-1} + k_t^T v_t,  o_t = q_t S_t.
 *   causal with the norm term (plain causal linear attention at gamma = 1):
 *            S_t = gamma S_{t-1} + f(k_t)^T v_t,  z_t = gamma z_{t-1} + f(k_t)
 *            o_t = f(q_t) S_t / (f(q_t) . z_t + eps),  f = phi or the identity.
 *
 * The backward formulas are derived by hand from those definitions (chain
 * rule, written out next to each function).  Every function works on one
 * (b,h) head at a time; heads are independent and are spread over
 * `nthreads` POSIX threads with a fixed head->thread assignment, so the
 * result does not depend on the thread count.
 *
 * Layout: every tensor is contiguous [B, H, T, D] (row-major, D fastest).
 * The optional bidir/simple `state` output is [B, H, D, D+1]: row i holds
 * S[i][0..D-1] followed by z[i] (z = 0 for simple).
 *
 * Return value: 0 on success, -1 on a bad argument or out of memory.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- phi -- */

/* elu(x) + 1 with elu's alpha = 1.  For x <= 0, elu(x) + 1 = exp(x) - 1 + 1
 * = exp(x); writing exp(x) directly avoids a cancellation. */
static double phi(double x) { return x > 0.0 ? x + 1.0 : exp(x); }

/* d/dx (elu(x) + 1): 1 for x > 0, exp(x) for x <= 0 (continuous at 0). */
static double dphi(double x) { return x > 0.0 ? 1.0 : exp(x); }

/* ------------------------------------------------------- head threading -- */

typedef struct {
    const double *q, *k, *v, *g;   /* g = upstream gradient dO (bwd only) */
    double *o, *state, *dq, *dk, *dv;
    const double *gamma;           /* [H] (retention only) */
    const double *state_in;        /* [B, H, D, D] state entering the sequence, or NULL (retention) */
    double *state_out;             /* [B, H, D, D] state after the last token, or NULL (retention fwd) */
    const double *dstate_in;       /* [B, H, D, D] R entering from after the sequence, or NULL (retention bwd) */
    double *dstate_out;            /* [B, H, D, D] R at the first token, or NULL (retention bwd) */
    long B, H, T, D;
    double eps;
    int use_phi, use_norm;
    int status;
} job_t;

typedef void (*head_fn)(job_t *job, long bh, double *scratch);

typedef struct {
    job_t *job;
    head_fn fn;
    long first, stride, nheads;
    size_t scratch_doubles;
    int failed;
} worker_t;

static void *worker_main(void *arg) {
    worker_t *w = (worker_t *)arg;
    double *scratch = (double *)malloc(w->scratch_doubles * sizeof(double));
    if (!scratch) { w->failed = 1; return NULL; }
    for (long bh = w->first; bh < w->nheads; bh += w->stride) w->fn(w->job, bh, scratch);
    free(scratch);
    return NULL;
}

/* Run fn over all B*H heads on nthreads threads (head bh -> thread bh % n). */
static int for_each_head(job_t *job, head_fn fn, size_t scratch_doubles, int nthreads) {
    long nheads = job->B * job->H;
    if (nthreads < 1) nthreads = 1;
    if (nthreads > nheads) nthreads = (int)(nheads > 0 ? nheads : 1);
    worker_t *ws = (worker_t *)calloc((size_t)nthreads, sizeof(worker_t));
    pthread_t *th = (pthread_t *)calloc((size_t)nthreads, sizeof(pthread_t));
    if (!ws || !th) { free(ws); free(th); return -1; }
    int rc = 0;
    for (int i = 0; i < nthreads; ++i) {
        ws[i].job = job; ws[i].fn = fn; ws[i].first = i; ws[i].stride = nthreads;
        ws[i].nheads = nheads; ws[i].scratch_doubles = scratch_doubles; ws[i].failed = 0;
    }
    int started = 0;
    for (int i = 1; i < nthreads; ++i) {
        if (pthread_create(&th[i], NULL, worker_main, &ws[i]) != 0) { ws[i].failed = 2; continue; }
        ++started;
    }
    worker_main(&ws[0]);
    for (int i = 1; i < nthreads; ++i)
        if (ws[i].failed != 2) pthread_join(th[i], NULL);
    for (int i = 0; i < nthreads; ++i) {
        if (ws[i].failed == 2) worker_main(&ws[i]);   /* thread could not start: run inline */
        if (ws[i].failed == 1) rc = -1;
    }
    (void)started;
    free(ws); free(th);
    return rc;
}

static int check_dims(long B, long H, long T, long D) {
    return (B >= 1 && H >= 1 && T >= 0 && D >= 1) ? 0 : -1;
}

/* ------------------------------------------- bidir / simple: forward ---- */

/* One head of the state form:
 *   S[i][j] = sum_s f(k_s)[i] v_s[j],   z[i] = sum_s f(k_s)[i]
 *   u_t[j]  = sum_i f(q_t)[i] S[i][j],  n_t = f(q_t) . z + eps
 *   o_t     = u_t / n_t        (norm on)      or   o_t = u_t  (norm off)
 * with f = phi (bidir) or the identity (simple). */
static void state_fwd_head(job_t *jb, long bh, double *scratch) {
    const long T = jb->T, D = jb->D;
    const double *q = jb->q + bh * T * D, *k = jb->k + bh * T * D, *v = jb->v + bh * T * D;
    double *o = jb->o + bh * T * D;
    double *S = scratch;            /* D*D */
    double *z = S + D * D;          /* D */
    double *fq = z + D;             /* D */
    memset(S, 0, (size_t)(D * D + D) * sizeof(double));
    for (long s = 0; s < T; ++s) {
        for (long i = 0; i < D; ++i) {
            double fk = jb->use_phi ? phi(k[s * D + i]) : k[s * D + i];
            z[i] += fk;
            for (long j = 0; j < D; ++j) S[i * D + j] += fk * v[s * D + j];
        }
    }
    for (long t = 0; t < T; ++t) {
        double n = jb->eps;
        for (long i = 0; i < D; ++i) {
            fq[i] = jb->use_phi ? phi(q[t * D + i]) : q[t * D + i];
            n += fq[i] * z[i];
        }
        for (long j = 0; j < D; ++j) {
            double u = 0.0;
            for (long i = 0; i < D; ++i) u += fq[i] * S[i * D + j];
            o[t * D + j] = jb->use_norm ? u / n : u;
        }
    }
    if (jb->state) {
        double *st = jb->state + bh * D * (D + 1);
        for (long i = 0; i < D; ++i) {
            for (long j = 0; j < D; ++j) st[i * (D + 1) + j] = S[i * D + j];
            st[i * (D + 1) + D] = jb->use_norm ? z[i] : 0.0;
        }
    }
}

/* ------------------------------------------ bidir / simple: backward ---- */

/* One head.  With g_t = dL/do_t and the forward quantities above:
 *   norm on:   dL/du_t = g_t / n_t,
 *              dL/dn_t = -(g_t . u_t) / n_t^2 = -(g_t . o_t) / n_t
 *              dfq_t   = (g_t S^T - (g_t . o_t) z) / n_t
 *              dS      = sum_t f(q_t)^T (g_t / n_t)
 *              dz      = -sum_t f(q_t) (g_t . o_t) / n_t
 *   norm off:  dfq_t = g_t S^T,  dS = sum_t q_t^T g_t,  dz = 0
 *   then       dfk_s = v_s dS^T + dz       (dfk_s[i] = sum_j dS[i][j] v_s[j] + dz[i])
 *              dv_s  = f(k_s) dS           (dv_s[j]  = sum_i f(k_s)[i] dS[i][j])
 *   and        dq = dfq * f'(q),  dk = dfk * f'(k)   (f' = dphi or 1). */
static void state_bwd_head(job_t *jb, long bh, double *scratch) {
    const long T = jb->T, D = jb->D;
    const long off = bh * T * D;
    const double *q = jb->q + off, *k = jb->k + off, *v = jb->v + off, *g = jb->g + off;
    double *dq = jb->dq + off, *dk = jb->dk + off, *dv = jb->dv + off;
    double *S = scratch, *z = S + D * D, *dS = z + D, *dz = dS + D * D, *fq = dz + D, *u = fq + D;
    memset(S, 0, (size_t)(2 * D * D + 2 * D) * sizeof(double));
    /* recompute S, z */
    for (long s = 0; s < T; ++s) {
        for (long i = 0; i < D; ++i) {
            double fk = jb->use_phi ? phi(k[s * D + i]) : k[s * D + i];
            z[i] += fk;
            for (long j = 0; j < D; ++j) S[i * D + j] += fk * v[s * D + j];
        }
    }
    /* query side: dq, and accumulate dS, dz */
    for (long t = 0; t < T; ++t) {
        double n = jb->eps;
        for (long i = 0; i < D; ++i) {
            fq[i] = jb->use_phi ? phi(q[t * D + i]) : q[t * D + i];
            n += fq[i] * z[i];
        }
        double go = 0.0;   /* g_t . o_t */
        for (long j = 0; j < D; ++j) {
            double uj = 0.0;
            for (long i = 0; i < D; ++i) uj += fq[i] * S[i * D + j];
            u[j] = uj;
            double oj = jb->use_norm ? uj / n : uj;
            go += g[t * D + j] * oj;
        }
        for (long i = 0; i < D; ++i) {
            double gs = 0.0;   /* (g_t S^T)[i] = sum_j g_t[j] S[i][j] */
            for (long j = 0; j < D; ++j) gs += g[t * D + j] * S[i * D + j];
            double dfq = jb->use_norm ? (gs - go * z[i]) / n : gs;
            double fp = jb->use_phi ? dphi(q[t * D + i]) : 1.0;
            dq[t * D + i] = dfq * fp;
            for (long j = 0; j < D; ++j)
                dS[i * D + j] += fq[i] * (jb->use_norm ? g[t * D + j] / n : g[t * D + j]);
            if (jb->use_norm) dz[i] -= fq[i] * go / n;
        }
    }
    /* key/value side */
    for (long s = 0; s < T; ++s) {
        for (long i = 0; i < D; ++i) {
            double a = dz[i];
            for (long j = 0; j < D; ++j) a += dS[i * D + j] * v[s * D + j];
            double fp = jb->use_phi ? dphi(k[s * D + i]) : 1.0;
            dk[s * D + i] = a * fp;
        }
        for (long j = 0; j < D; ++j) {
            double a = 0.0;
            for (long i = 0; i < D; ++i) {
                double fk = jb->use_phi ? phi(k[s * D + i]) : k[s * D + i];
                a += fk * dS[i * D + j];
            }
            dv[s * D + j] = a;
        }
    }
}

int oracle_bidir_fwd(const double *q, const double *k, const double *v, double *o, double *state,
                     long B, long H, long T, long D, double eps, int nthreads) {
    if (check_dims(B, H, T, D) || !q || !k || !v || !o) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.o = o; jb.state = state;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D; jb.eps = eps; jb.use_phi = 1; jb.use_norm = 1;
    return for_each_head(&jb, state_fwd_head, (size_t)(D * D + 2 * D), nthreads);
}

int oracle_simple_fwd(const double *q, const double *k, const double *v, double *o, double *state,
                      long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || !q || !k || !v || !o) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.o = o; jb.state = state;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D; jb.eps = 0.0; jb.use_phi = 0; jb.use_norm = 0;
    return for_each_head(&jb, state_fwd_head, (size_t)(D * D + 2 * D), nthreads);
}

int oracle_bidir_bwd(const double *q, const double *k, const double *v, const double *dout,
                     double *dq, double *dk, double *dv,
                     long B, long H, long T, long D, double eps, int nthreads) {
    if (check_dims(B, H, T, D) || !q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.g = dout; jb.dq = dq; jb.dk = dk; jb.dv = dv;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D; jb.eps = eps; jb.use_phi = 1; jb.use_norm = 1;
    return for_each_head(&jb, state_bwd_head, (size_t)(2 * D * D + 4 * D), nthreads);
}

int oracle_simple_bwd(const double *q, const double *k, const double *v, const double *dout,
                      double *dq, double *dk, double *dv,
                      long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || !q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.g = dout; jb.dq = dq; jb.dk = dk; jb.dv = dv;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D; jb.eps = 0.0; jb.use_phi = 0; jb.use_norm = 0;
    return for_each_head(&jb, state_bwd_head, (size_t)(2 * D * D + 4 * D), nthreads);
}

/* ------------------------------------------------ retention (recurrent) -- */

/* Forward, one head, the recurrent form:
 *   S_t = gamma S_{t-1} + k_t^T v_t   (S_{-1} = 0),   o_t = q_t S_t. */
static void retention_fwd_head(job_t *jb, long bh, double *scratch) {
    const long T = jb->T, D = jb->D;
    const double gamma = jb->gamma[bh % jb->H];
    const long off = bh * T * D;
    const double *q = jb->q + off, *k = jb->k + off, *v = jb->v + off;
    double *o = jb->o + off;
    double *S = scratch;
    if (jb->state_in)
        memcpy(S, jb->state_in + bh * D * D, (size_t)(D * D) * sizeof(double));
    else
        memset(S, 0, (size_t)(D * D) * sizeof(double));
    for (long t = 0; t < T; ++t) {
        for (long i = 0; i < D; ++i)
            for (long j = 0; j < D; ++j)
                S[i * D + j] = gamma * S[i * D + j] + k[t * D + i] * v[t * D + j];
        for (long j = 0; j < D; ++j) {
            double a = 0.0;
            for (long i = 0; i < D; ++i) a += q[t * D + i] * S[i * D + j];
            o[t * D + j] = a;
        }
    }
    if (jb->state_out) memcpy(jb->state_out + bh * D * D, S, (size_t)(D * D) * sizeof(double));
}

/* Backward, one head.
 *   dq_t[i] = sum_j S_t[i][j] g_t[j]                        (forward sweep)
 *   R_t     = gamma R_{t+1} + q_t^T g_t   (R_T = 0)          (reverse sweep)
 *             i.e. R_s = sum_{t>=s} gamma^(t-s) q_t^T g_t
 *   dk_s[i] = sum_j R_s[i][j] v_s[j],   dv_s[j] = sum_i k_s[i] R_s[i][j].
 * For a segment of a longer sequence S_{-1} = state_in (the tokens before it) and
 * R_T = dstate_in (the tokens after it) instead of zero; R_0 goes to dstate_out. */
static void retention_bwd_head(job_t *jb, long bh, double *scratch) {
    const long T = jb->T, D = jb->D;
    const double gamma = jb->gamma[bh % jb->H];
    const long off = bh * T * D;
    const double *q = jb->q + off, *k = jb->k + off, *v = jb->v + off, *g = jb->g + off;
    double *dq = jb->dq + off, *dk = jb->dk + off, *dv = jb->dv + off;
    double *S = scratch, *R = S + D * D;
    memset(S, 0, (size_t)(2 * D * D) * sizeof(double));
    if (jb->state_in) memcpy(S, jb->state_in + bh * D * D, (size_t)(D * D) * sizeof(double));
    if (jb->dstate_in) memcpy(R, jb->dstate_in + bh * D * D, (size_t)(D * D) * sizeof(double));
    for (long t = 0; t < T; ++t) {
        for (long i = 0; i < D; ++i)
            for (long j = 0; j < D; ++j)
                S[i * D + j] = gamma * S[i * D + j] + k[t * D + i] * v[t * D + j];
        for (long i = 0; i < D; ++i) {
            double a = 0.0;
            for (long j = 0; j < D; ++j) a += S[i * D + j] * g[t * D + j];
            dq[t * D + i] = a;
        }
    }
    for (long s = T - 1; s >= 0; --s) {
        for (long i = 0; i < D; ++i)
            for (long j = 0; j < D; ++j)
                R[i * D + j] = gamma * R[i * D + j] + q[s * D + i] * g[s * D + j];
        for (long i = 0; i < D; ++i) {
            double a = 0.0;
            for (long j = 0; j < D; ++j) a += R[i * D + j] * v[s * D + j];
            dk[s * D + i] = a;
        }
        for (long j = 0; j < D; ++j) {
            double a = 0.0;
            for (long i = 0; i < D; ++i) a += k[s * D + i] * R[i * D + j];
            dv[s * D + j] = a;
        }
    }
    if (jb->dstate_out) memcpy(jb->dstate_out + bh * D * D, R, (size_t)(D * D) * sizeof(double));
}

int oracle_retention_fwd(const double *q, const double *k, const double *v, const double *gamma,
                         double *o, long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || !q || !k || !v || !gamma || !o) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.gamma = gamma; jb.o = o;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D;
    return for_each_head(&jb, retention_fwd_head, (size_t)(D * D), nthreads);
}

/* One recurrent step of retention (decode), every head (the FusedRecurrent
 * update applied to a single token):
 *   S <- gamma_h S + k^T v,    o = q S
 * q, k, v, o are [B, H, D]; S is [B, H, D, D] (row i = key index i, column j =
 * value index j) and is updated in place. */
int oracle_retention_step(const double *q, const double *k, const double *v, const double *gamma,
                          double *S, double *o, long B, long H, long D) {
    if (B < 1 || H < 1 || D < 1 || !q || !k || !v || !gamma || !S || !o) return -1;
    for (long bh = 0; bh < B * H; ++bh) {
        const double g = gamma[bh % H];
        const double *qh = q + bh * D, *kh = k + bh * D, *vh = v + bh * D;
        double *Sh = S + bh * D * D, *oh = o + bh * D;
        for (long i = 0; i < D; ++i)
            for (long j = 0; j < D; ++j)
                Sh[i * D + j] = g * Sh[i * D + j] + kh[i] * vh[j];
        for (long j = 0; j < D; ++j) {
            double a = 0.0;
            for (long i = 0; i < D; ++i) a += qh[i] * Sh[i * D + j];
            oh[j] = a;
        }
    }
    return 0;
}

/* oracle_retention_fwd from a given state: S starts at state_in (zero if NULL)
 * instead of zero, and the state after the last token goes to state_out (if not
 * NULL).  Arrays [B, H, D, D]. */
int oracle_retention_fwd_state(const double *q, const double *k, const double *v, const double *gamma,
                               const double *state_in, double *o, double *state_out,
                               long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || (T > 0 && (!q || !k || !v || !o)) || !gamma) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.gamma = gamma; jb.o = o;
    jb.state_in = state_in; jb.state_out = state_out;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D;
    return for_each_head(&jb, retention_fwd_head, (size_t)(D * D), nthreads);
}

int oracle_retention_bwd(const double *q, const double *k, const double *v, const double *dout,
                         const double *gamma, double *dq, double *dk, double *dv,
                         long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || !q || !k || !v || !dout || !gamma || !dq || !dk || !dv) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.g = dout; jb.gamma = gamma; jb.dq = dq; jb.dk = dk; jb.dv = dv;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D;
    return for_each_head(&jb, retention_bwd_head, (size_t)(2 * D * D), nthreads);
}

/* oracle_retention_bwd of one segment of a longer sequence: state_in is the state
 * of the tokens before it, dstate_in the reverse-sweep R of the tokens after it
 * (both zero if NULL); R at the segment's first token goes to dstate_out (if not
 * NULL).  Arrays [B, H, D, D]. */
int oracle_retention_bwd_state(const double *q, const double *k, const double *v, const double *dout,
                               const double *gamma, const double *state_in, const double *dstate_in,
                               double *dq, double *dk, double *dv, double *dstate_out,
                               long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || (T > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv)) || !gamma) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.g = dout; jb.gamma = gamma; jb.dq = dq; jb.dk = dk; jb.dv = dv;
    jb.state_in = state_in; jb.dstate_in = dstate_in; jb.dstate_out = dstate_out;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D;
    return for_each_head(&jb, retention_bwd_head, (size_t)(2 * D * D), nthreads);
}

/* ------------------------------------- causal with the norm term (recurrent) -- */

static double feat(const job_t *jb, double x) { return jb->use_phi ? phi(x) : x; }
static double dfeat(const job_t *jb, double x) { return jb->use_phi ? dphi(x) : 1.0; }
static double head_gamma(const job_t *jb, long bh) { return jb->gamma ? jb->gamma[bh % jb->H] : 1.0; }

/* Forward, one head:
 *   S_t = gamma S_{t-1} + f(k_t)^T v_t,  z_t = gamma z_{t-1} + f(k_t)   (S_{-1} = 0, z_{-1} = 0)
 *   o_t = f(q_t) S_t / (f(q_t) . z_t + eps). */
static void causal_fwd_head(job_t *jb, long bh, double *scratch) {
    const long T = jb->T, D = jb->D;
    const double gamma = head_gamma(jb, bh);
    const long off = bh * T * D;
    const double *q = jb->q + off, *k = jb->k + off, *v = jb->v + off;
    double *o = jb->o + off;
    double *S = scratch, *z = S + D * D, *fq = z + D, *fk = fq + D;
    memset(S, 0, (size_t)(D * D + D) * sizeof(double));
    for (long t = 0; t < T; ++t) {
        for (long i = 0; i < D; ++i) {
            fq[i] = feat(jb, q[t * D + i]);
            fk[i] = feat(jb, k[t * D + i]);
        }
        for (long i = 0; i < D; ++i) {
            z[i] = gamma * z[i] + fk[i];
            for (long j = 0; j < D; ++j) S[i * D + j] = gamma * S[i * D + j] + fk[i] * v[t * D + j];
        }
        double n = jb->eps;
        for (long i = 0; i < D; ++i) n += fq[i] * z[i];
        for (long j = 0; j < D; ++j) {
            double u = 0.0;
            for (long i = 0; i < D; ++i) u += fq[i] * S[i * D + j];
            o[t * D + j] = u / n;
        }
    }
}

/* Backward, one head.  With u_t = f(q_t) S_t, n_t = f(q_t) . z_t + eps, o_t = u_t / n_t:
 *   du_t = dout_t / n_t,   dn_t = -(dout_t . o_t) / n_t
 *   df(q)_t[i] = sum_j S_t[i][j] du_t[j] + z_t[i] dn_t                     (forward sweep)
 *   R_s = gamma R_{s+1} + f(q_s)^T du_s,   r_s = gamma r_{s+1} + f(q_s) dn_s  (reverse sweep)
 *   df(k)_s[i] = sum_j R_s[i][j] v_s[j] + r_s[i],   dv_s[j] = sum_i f(k_s)[i] R_s[i][j]
 *   dq = df(q) f'(q),  dk = df(k) f'(k). */
static void causal_bwd_head(job_t *jb, long bh, double *scratch) {
    const long T = jb->T, D = jb->D;
    const double gamma = head_gamma(jb, bh);
    const long off = bh * T * D;
    const double *q = jb->q + off, *k = jb->k + off, *v = jb->v + off, *g = jb->g + off;
    double *dq = jb->dq + off, *dk = jb->dk + off, *dv = jb->dv + off;
    double *S = scratch, *z = S + D * D, *R = z + D, *r = R + D * D, *fq = r + D, *fk = fq + D;
    double *nt = fk + D, *dnt = nt + T;            /* n_t and dn_t of every row */
    memset(S, 0, (size_t)(2 * D * D + 2 * D) * sizeof(double));
    for (long t = 0; t < T; ++t) {
        for (long i = 0; i < D; ++i) {
            fq[i] = feat(jb, q[t * D + i]);
            fk[i] = feat(jb, k[t * D + i]);
        }
        for (long i = 0; i < D; ++i) {
            z[i] = gamma * z[i] + fk[i];
            for (long j = 0; j < D; ++j) S[i * D + j] = gamma * S[i * D + j] + fk[i] * v[t * D + j];
        }
        double n = jb->eps;
        for (long i = 0; i < D; ++i) n += fq[i] * z[i];
        double go = 0.0;                          /* dout_t . o_t */
        for (long j = 0; j < D; ++j) {
            double u = 0.0;
            for (long i = 0; i < D; ++i) u += fq[i] * S[i * D + j];
            go += g[t * D + j] * (u / n);
        }
        const double dn = -go / n;
        nt[t] = n;
        dnt[t] = dn;
        for (long i = 0; i < D; ++i) {
            double a = z[i] * dn;
            for (long j = 0; j < D; ++j) a += S[i * D + j] * (g[t * D + j] / n);
            dq[t * D + i] = a * dfeat(jb, q[t * D + i]);
        }
    }
    for (long s = T - 1; s >= 0; --s) {
        for (long i = 0; i < D; ++i) {
            fq[i] = feat(jb, q[s * D + i]);
            fk[i] = feat(jb, k[s * D + i]);
        }
        for (long i = 0; i < D; ++i) {
            r[i] = gamma * r[i] + fq[i] * dnt[s];
            for (long j = 0; j < D; ++j) R[i * D + j] = gamma * R[i * D + j] + fq[i] * (g[s * D + j] / nt[s]);
        }
        for (long i = 0; i < D; ++i) {
            double a = r[i];
            for (long j = 0; j < D; ++j) a += R[i * D + j] * v[s * D + j];
            dk[s * D + i] = a * dfeat(jb, k[s * D + i]);
        }
        for (long j = 0; j < D; ++j) {
            double a = 0.0;
            for (long i = 0; i < D; ++i) a += fk[i] * R[i * D + j];
            dv[s * D + j] = a;
        }
    }
}

/* gamma: [H] decays in (0, 1], or NULL for gamma = 1.  use_phi: 1 = elu + 1, 0 = identity. */
int oracle_causal_norm_fwd(const double *q, const double *k, const double *v, const double *gamma, int use_phi,
                           double eps, double *o, long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || (T > 0 && (!q || !k || !v || !o))) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.gamma = gamma; jb.o = o; jb.use_phi = use_phi; jb.use_norm = 1; jb.eps = eps;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D;
    return for_each_head(&jb, causal_fwd_head, (size_t)(D * D + 3 * D), nthreads);
}

int oracle_causal_norm_bwd(const double *q, const double *k, const double *v, const double *dout,
                           const double *gamma, int use_phi, double eps, double *dq, double *dk, double *dv,
                           long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || (T > 0 && (!q || !k || !v || !dout || !dq || !dk || !dv))) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.g = dout; jb.gamma = gamma; jb.dq = dq; jb.dk = dk; jb.dv = dv;
    jb.use_phi = use_phi; jb.use_norm = 1; jb.eps = eps;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D;
    return for_each_head(&jb, causal_bwd_head, (size_t)(2 * D * D + 4 * D + 2 * T), nthreads);
}

/* --------------------- bidirectional with the norm term on given features -- */

/* la_bidir's definition with f the identity: q, k are features the caller formed. */
int oracle_normed_fwd(const double *q, const double *k, const double *v, double *o, double *state,
                      long B, long H, long T, long D, double eps, int nthreads) {
    if (check_dims(B, H, T, D) || !q || !k || !v || !o) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.o = o; jb.state = state;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D; jb.eps = eps; jb.use_phi = 0; jb.use_norm = 1;
    return for_each_head(&jb, state_fwd_head, (size_t)(D * D + 2 * D), nthreads);
}

int oracle_normed_bwd(const double *q, const double *k, const double *v, const double *dout,
                      double *dq, double *dk, double *dv,
                      long B, long H, long T, long D, double eps, int nthreads) {
    if (check_dims(B, H, T, D) || !q || !k || !v || !dout || !dq || !dk || !dv) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.g = dout; jb.dq = dq; jb.dk = dk; jb.dv = dv;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D; jb.eps = eps; jb.use_phi = 0; jb.use_norm = 1;
    return for_each_head(&jb, state_bwd_head, (size_t)(2 * D * D + 4 * D), nthreads);
}

/* ----------------------------------------------------- feature maps, per row -- */

/* kind 0, the focusing function of focused linear attention: with y = relu(x),
 *   f(x) = (|y| / |y^p|) y^p      (|.| the 2-norm of the row, y^p elementwise; 0 if y = 0),
 * so the row keeps the norm of relu(x) while its direction sharpens towards the
 * largest entries.  Kinds 1 and 2, the polarity split: f(x) = [relu(x)^p, relu(-x)^p]
 * (kind 1) or [relu(-x)^p, relu(x)^p] (kind 2), twice the width of x. */
static int fmap_width(int kind, long D) { return kind == 0 ? (int)D : (int)(2 * D); }

static void fmap_row_fwd(int kind, double p, const double *x, double *y, long D) {
    if (kind == 0) {
        double a = 0.0, b = 0.0;
        for (long i = 0; i < D; ++i) {
            const double r = x[i] > 0.0 ? x[i] : 0.0;
            a += r * r;
            b += pow(r, 2.0 * p);
        }
        a = sqrt(a);
        b = sqrt(b);
        for (long i = 0; i < D; ++i) {
            const double r = x[i] > 0.0 ? x[i] : 0.0;
            y[i] = b > 0.0 ? (a / b) * pow(r, p) : 0.0;
        }
        return;
    }
    for (long i = 0; i < D; ++i) {
        const double pos = x[i] > 0.0 ? pow(x[i], p) : 0.0, neg = x[i] < 0.0 ? pow(-x[i], p) : 0.0;
        y[i] = kind == 1 ? pos : neg;
        y[D + i] = kind == 1 ? neg : pos;
    }
}

/* dx = J^T dy, J the Jacobian of the row's map.  Focusing function, with a = |y|,
 * b = |y^p|, u = y^p and s = dy . u (y = relu(x)):
 *   dx_j = [x_j > 0] ((a / b) p y_j^(p-1) dy_j + s y_j / (a b) - s a p y_j^(2p-1) / b^3).
 * Polarity split: d relu(x)^p / dx = p x^(p-1) [x > 0], d relu(-x)^p / dx = -p (-x)^(p-1) [x < 0]. */
static void fmap_row_bwd(int kind, double p, const double *x, const double *dy, double *dx, long D) {
    if (kind == 0) {
        double a = 0.0, b = 0.0, s = 0.0;
        for (long i = 0; i < D; ++i) {
            const double r = x[i] > 0.0 ? x[i] : 0.0;
            a += r * r;
            b += pow(r, 2.0 * p);
            s += dy[i] * pow(r, p);
        }
        a = sqrt(a);
        b = sqrt(b);
        for (long j = 0; j < D; ++j) {
            if (!(x[j] > 0.0) || b <= 0.0) { dx[j] = 0.0; continue; }
            const double r = x[j];
            dx[j] = (a / b) * p * pow(r, p - 1.0) * dy[j] + s * r / (a * b) - s * a * p * pow(r, 2.0 * p - 1.0) / (b * b * b);
        }
        return;
    }
    for (long i = 0; i < D; ++i) {
        const double dpos = x[i] > 0.0 ? p * pow(x[i], p - 1.0) : 0.0;
        const double dneg = x[i] < 0.0 ? -p * pow(-x[i], p - 1.0) : 0.0;
        const double gpos = kind == 1 ? dy[i] : dy[D + i], gneg = kind == 1 ? dy[D + i] : dy[i];
        dx[i] = gpos * dpos + gneg * dneg;
    }
}

/* x [rows, D] -> y [rows, width]; p > 0. */
int oracle_feature_map_fwd(int kind, double p, const double *x, double *y, long rows, long D) {
    if (kind < 0 || kind > 2 || !(p > 0.0) || rows < 0 || D < 1 || (rows > 0 && (!x || !y))) return -1;
    const long w = fmap_width(kind, D);
    for (long r = 0; r < rows; ++r) fmap_row_fwd(kind, p, x + r * D, y + r * w, D);
    return 0;
}

int oracle_feature_map_bwd(int kind, double p, const double *x, const double *dy, double *dx, long rows, long D) {
    if (kind < 0 || kind > 2 || !(p > 0.0) || rows < 0 || D < 1 || (rows > 0 && (!x || !dy || !dx))) return -1;
    const long w = fmap_width(kind, D);
    for (long r = 0; r < rows; ++r) fmap_row_bwd(kind, p, x + r * D, dy + r * w, dx + r * D, D);
    return 0;
}

/* ------------------------------------------ gated linear attention (recurrent) -- */

/* Forward, one head: S_t[i][j] = exp(g_t[i]) S_{t-1}[i][j] + k_t[i] v_t[j], o_t = q_t S_t. */
static void gated_fwd_head(job_t *jb, long bh, double *scratch) {
    const long T = jb->T, D = jb->D;
    const long off = bh * T * D;
    const double *q = jb->q + off, *k = jb->k + off, *v = jb->v + off, *lg = jb->state_in + off;
    double *o = jb->o + off;
    double *S = scratch;
    memset(S, 0, (size_t)(D * D) * sizeof(double));
    for (long t = 0; t < T; ++t) {
        for (long i = 0; i < D; ++i) {
            const double a = exp(lg[t * D + i]);
            for (long j = 0; j < D; ++j) S[i * D + j] = a * S[i * D + j] + k[t * D + i] * v[t * D + j];
        }
        for (long j = 0; j < D; ++j) {
            double u = 0.0;
            for (long i = 0; i < D; ++i) u += q[t * D + i] * S[i * D + j];
            o[t * D + j] = u;
        }
    }
}

/* Backward, one head.
 *   dq_t[i] = sum_j S_t[i][j] dout_t[j]                                   (forward sweep)
 *   R_t = q_t^T dout_t + diag(exp(g_{t+1})) R_{t+1}  (R_T = 0)            (reverse sweep)
 *   dk_t[i] = sum_j R_t[i][j] v_t[j],   dv_t[j] = sum_i k_t[i] R_t[i][j]
 * and the log gates: with G_t = sum_{s<=t} g_s, o_t = sum_{s<=t} (q_t e^{G_t}) . (k_s e^{-G_s}) v_s,
 * so dL/dG_t = q_t dq_t - k_t dk_t (elementwise) and dg_t = sum_{s>=t} (q_s dq_s - k_s dk_s). */
static void gated_bwd_head(job_t *jb, long bh, double *scratch) {
    const long T = jb->T, D = jb->D;
    const long off = bh * T * D;
    const double *q = jb->q + off, *k = jb->k + off, *v = jb->v + off, *g = jb->g + off, *lg = jb->state_in + off;
    double *dq = jb->dq + off, *dk = jb->dk + off, *dv = jb->dv + off, *dg = jb->state_out + off;
    double *S = scratch, *R = S + D * D, *acc = R + D * D;
    memset(S, 0, (size_t)(2 * D * D + D) * sizeof(double));
    for (long t = 0; t < T; ++t) {
        for (long i = 0; i < D; ++i) {
            const double a = exp(lg[t * D + i]);
            for (long j = 0; j < D; ++j) S[i * D + j] = a * S[i * D + j] + k[t * D + i] * v[t * D + j];
        }
        for (long i = 0; i < D; ++i) {
            double a = 0.0;
            for (long j = 0; j < D; ++j) a += S[i * D + j] * g[t * D + j];
            dq[t * D + i] = a;
        }
    }
    for (long t = T - 1; t >= 0; --t) {
        for (long i = 0; i < D; ++i) {
            const double a = t + 1 < T ? exp(lg[(t + 1) * D + i]) : 0.0;
            for (long j = 0; j < D; ++j) R[i * D + j] = a * R[i * D + j] + q[t * D + i] * g[t * D + j];
        }
        for (long i = 0; i < D; ++i) {
            double a = 0.0;
            for (long j = 0; j < D; ++j) a += R[i * D + j] * v[t * D + j];
            dk[t * D + i] = a;
        }
        for (long j = 0; j < D; ++j) {
            double a = 0.0;
            for (long i = 0; i < D; ++i) a += k[t * D + i] * R[i * D + j];
            dv[t * D + j] = a;
        }
    }
    for (long t = T - 1; t >= 0; --t)
        for (long i = 0; i < D; ++i) {
            acc[i] += q[t * D + i] * dq[t * D + i] - k[t * D + i] * dk[t * D + i];
            dg[t * D + i] = acc[i];
        }
}

/* lg: [B, H, T, D] log gates (<= 0 for a decay); dg: their gradient. */
int oracle_gated_fwd(const double *q, const double *k, const double *v, const double *lg, double *o,
                     long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || (T > 0 && (!q || !k || !v || !lg || !o))) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.state_in = lg; jb.o = o;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D;
    return for_each_head(&jb, gated_fwd_head, (size_t)(D * D), nthreads);
}

int oracle_gated_bwd(const double *q, const double *k, const double *v, const double *lg, const double *dout,
                     double *dq, double *dk, double *dv, double *dg, long B, long H, long T, long D, int nthreads) {
    if (check_dims(B, H, T, D) || (T > 0 && (!q || !k || !v || !lg || !dout || !dq || !dk || !dv || !dg))) return -1;
    job_t jb; memset(&jb, 0, sizeof jb);
    jb.q = q; jb.k = k; jb.v = v; jb.state_in = lg; jb.g = dout; jb.dq = dq; jb.dk = dk; jb.dv = dv; jb.state_out = dg;
    jb.B = B; jb.H = H; jb.T = T; jb.D = D;
    return for_each_head(&jb, gated_bwd_head, (size_t)(2 * D * D + D), nthreads);
}


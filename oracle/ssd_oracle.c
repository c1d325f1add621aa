/*
 * ssd_oracle.c -- fp64 CPU oracle for the Mamba-2 SSD forward scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the CPU-baseline leg of the
 * benchmark do.  It shares no code, header or table with the CUDA library.
 *
 * What is computed (per batch b and head h, with group g = h / (H/G)):
 *
 *   h_t = exp(dt_t * A_h) * h_{t-1} + dt_t * x_t B_t^T        (P x N state)
 *   y_t = h_t C_t + D_h * x_t
 *
 * This is the selective SSM recurrence with a scalar-times-identity transition
 * A_t = a_t I ("Transformers are SSMs", Dao & Gu 2024, as summarised on
 * akillness.github.io "State Space Duality and Mamba-2", section "Mathematical
 * Foundations" and "The Scalar-Identity Structural Constraint"), with the step
 * size dt entering as a_t = exp(dt_t A_h) on the state and dt_t on the input.
 * The skip term D_h x_t is added to every output.
 *
 * Three independent evaluations are provided:
 *   oracle_ssd_recurrent  -- the token-by-token recurrence above (the oracle).
 *   oracle_ssd_quadratic  -- the dual "attention" form y = M x with the explicit
 *                            T x T semiseparable matrix
 *                            M[t][s] = C_t . B_s * dt_s * prod_{k=s+1..t} a_k
 *                            (akillness.github.io, "Mathematical Foundations",
 *                            the 3x3 matrix and the unrolled product), used
 *                            only to pin the recurrence on small T.
 *   oracle_ssd_chunked    -- the chunked algorithm (aifetchly blog, "The
 *                            Chunked SSD Algorithm", steps 1-2; d-central
 *                            glossary, "Why it is useful": attention inside
 *                            chunks, recurrence between them), written with the
 *                            cumulative log-decay of akillness.github.io ("The
 *                            Scalar-Identity Structural Constraint": the decay
 *                            between i and j is exp(s_j - s_i)).  It can also
 *                            return every intermediate of the four stages.
 *
 * Layouts (all row-major, contiguous, fp64):
 *   x, y        [B, T, H, P]
 *   dt          [B, T, H]
 *   A, D        [H]            (D may be NULL: no skip term)
 *   Bm, Cm      [B, T, G, N]
 *   h0, final   [B, H, P, N]   (h0 may be NULL: zero initial state;
 *                               final may be NULL: not written)
 */
#define _GNU_SOURCE
#include <math.h>
#include <pthread.h>
#include <sched.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

typedef struct {
    int64_t batch, seqlen, nheads, headdim, dstate, ngroups;
} oracle_dims_t;

typedef struct {
    const oracle_dims_t *d;
    const double *x, *dt, *A, *Bm, *Cm, *D, *h0;
    double *y, *final_state;
    const int64_t *units; /* list of (b*H + h) to evaluate; NULL = all */
    int64_t nunits;
    int64_t next; /* work counter */
} rec_job_t;

static inline int64_t idx_x(const oracle_dims_t *d, int64_t b, int64_t t, int64_t h, int64_t p) {
    return ((b * d->seqlen + t) * d->nheads + h) * d->headdim + p;
}
static inline int64_t idx_dt(const oracle_dims_t *d, int64_t b, int64_t t, int64_t h) {
    return (b * d->seqlen + t) * d->nheads + h;
}
static inline int64_t idx_bc(const oracle_dims_t *d, int64_t b, int64_t t, int64_t g, int64_t n) {
    return ((b * d->seqlen + t) * d->ngroups + g) * d->dstate + n;
}
static inline int64_t idx_st(const oracle_dims_t *d, int64_t b, int64_t h, int64_t p, int64_t n) {
    return ((b * d->nheads + h) * d->headdim + p) * d->dstate + n;
}
static inline int64_t group_of(const oracle_dims_t *d, int64_t h) {
    return h / (d->nheads / d->ngroups);
}

/* ------------------------------------------------------------------------- */
/* Recurrent form: one (b, h) unit, token by token.                          */
/* ------------------------------------------------------------------------- */
static void recurrent_unit(const rec_job_t *j, int64_t unit, double *S) {
    const oracle_dims_t *d = j->d;
    const int64_t b = unit / d->nheads, h = unit % d->nheads, g = group_of(d, h);
    const int64_t P = d->headdim, N = d->dstate;
    for (int64_t p = 0; p < P; ++p)
        for (int64_t n = 0; n < N; ++n)
            S[p * N + n] = j->h0 ? j->h0[idx_st(d, b, h, p, n)] : 0.0;
    const double Dh = j->D ? j->D[h] : 0.0;
    for (int64_t t = 0; t < d->seqlen; ++t) {
        const double dt = j->dt[idx_dt(d, b, t, h)];
        const double a = exp(dt * j->A[h]);
        const double *xt = j->x + idx_x(d, b, t, h, 0);
        const double *Bt = j->Bm + idx_bc(d, b, t, g, 0);
        const double *Ct = j->Cm + idx_bc(d, b, t, g, 0);
        double *yt = j->y + idx_x(d, b, t, h, 0);
        for (int64_t p = 0; p < P; ++p) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n) {
                S[p * N + n] = a * S[p * N + n] + dt * xt[p] * Bt[n];
                acc += S[p * N + n] * Ct[n];
            }
            yt[p] = acc + Dh * xt[p];
        }
    }
    if (j->final_state)
        for (int64_t p = 0; p < P; ++p)
            for (int64_t n = 0; n < N; ++n)
                j->final_state[idx_st(d, b, h, p, n)] = S[p * N + n];
}

static void *recurrent_worker(void *arg) {
    rec_job_t *j = (rec_job_t *)arg;
    double *S = (double *)malloc(sizeof(double) * j->d->headdim * j->d->dstate);
    if (!S) return NULL;
    for (;;) {
        int64_t k = __atomic_fetch_add(&j->next, 1, __ATOMIC_RELAXED);
        if (k >= j->nunits) break;
        recurrent_unit(j, j->units ? j->units[k] : k, S);
    }
    free(S);
    return NULL;
}

int oracle_default_threads(void) {
    cpu_set_t set;
    if (sched_getaffinity(0, sizeof(set), &set) == 0) return CPU_COUNT(&set);
    return 1;
}

/* Evaluate the recurrence for the listed (b, h) units (units == NULL: all B*H
 * units).  Outputs are written only for those units.  nthreads <= 0 uses every
 * core in the affinity mask.  Returns 0 on success, negative on bad input. */
int oracle_ssd_recurrent(const oracle_dims_t *d, const double *x, const double *dt,
                         const double *A, const double *Bm, const double *Cm,
                         const double *D, const double *h0, double *y,
                         double *final_state, const int64_t *units, int64_t nunits,
                         int nthreads) {
    if (!d || !x || !dt || !A || !Bm || !Cm || !y) return -1;
    if (d->ngroups <= 0 || d->nheads % d->ngroups != 0) return -2;
    rec_job_t job = {d, x, dt, A, Bm, Cm, D, h0, y, final_state, units,
                     units ? nunits : d->batch * d->nheads, 0};
    if (nthreads <= 0) nthreads = oracle_default_threads();
    if (nthreads > job.nunits) nthreads = (int)(job.nunits > 0 ? job.nunits : 1);
    if (nthreads == 1) {
        recurrent_worker(&job);
        return 0;
    }
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    if (!th) return -3;
    int started = 0;
    for (int i = 0; i < nthreads; ++i)
        if (pthread_create(&th[i], NULL, recurrent_worker, &job) == 0) ++started;
    if (started == 0) recurrent_worker(&job);
    for (int i = 0; i < started; ++i) pthread_join(th[i], NULL);
    free(th);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Quadratic (dual) form with the explicit T x T matrix, for small T.        */
/* M[t][s] = (C_t . B_s) * dt_s * prod_{k=s+1}^{t} exp(dt_k A_h), s <= t.    */
/* The initial state reaches y_t through prod_{k=0}^{t} exp(dt_k A_h).       */
/* ------------------------------------------------------------------------- */
int oracle_ssd_quadratic(const oracle_dims_t *d, const double *x, const double *dt,
                         const double *A, const double *Bm, const double *Cm,
                         const double *D, const double *h0, double *y,
                         double *final_state) {
    if (!d || !x || !dt || !A || !Bm || !Cm || !y) return -1;
    if (d->ngroups <= 0 || d->nheads % d->ngroups != 0) return -2;
    const int64_t T = d->seqlen, P = d->headdim, N = d->dstate;
    double *M = (double *)malloc(sizeof(double) * T * T);
    double *decay0 = (double *)malloc(sizeof(double) * T); /* prod_{k=0}^{t} a_k */
    double *a = (double *)malloc(sizeof(double) * T);
    if (!M || !decay0 || !a) {
        free(M); free(decay0); free(a);
        return -3;
    }
    for (int64_t b = 0; b < d->batch; ++b)
        for (int64_t h = 0; h < d->nheads; ++h) {
            const int64_t g = group_of(d, h);
            for (int64_t t = 0; t < T; ++t) a[t] = exp(dt[idx_dt(d, b, t, h)] * A[h]);
            for (int64_t t = 0; t < T; ++t) {
                double pr = 1.0;
                for (int64_t k = 0; k <= t; ++k) pr *= a[k];
                decay0[t] = pr;
                for (int64_t s = 0; s < T; ++s) {
                    if (s > t) { M[t * T + s] = 0.0; continue; }
                    double prod = 1.0;
                    for (int64_t k = s + 1; k <= t; ++k) prod *= a[k];
                    double cb = 0.0;
                    for (int64_t n = 0; n < N; ++n)
                        cb += Cm[idx_bc(d, b, t, g, n)] * Bm[idx_bc(d, b, s, g, n)];
                    M[t * T + s] = cb * dt[idx_dt(d, b, s, h)] * prod;
                }
            }
            for (int64_t t = 0; t < T; ++t)
                for (int64_t p = 0; p < P; ++p) {
                    double acc = 0.0;
                    for (int64_t s = 0; s <= t; ++s) acc += M[t * T + s] * x[idx_x(d, b, s, h, p)];
                    if (h0) {
                        double hc = 0.0;
                        for (int64_t n = 0; n < N; ++n)
                            hc += h0[idx_st(d, b, h, p, n)] * Cm[idx_bc(d, b, t, g, n)];
                        acc += decay0[t] * hc;
                    }
                    if (D) acc += D[h] * x[idx_x(d, b, t, h, p)];
                    y[idx_x(d, b, t, h, p)] = acc;
                }
            if (final_state)
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n) {
                        double acc = h0 ? decay0[T - 1] * h0[idx_st(d, b, h, p, n)] : 0.0;
                        for (int64_t s = 0; s < T; ++s) {
                            double prod = 1.0;
                            for (int64_t k = s + 1; k < T; ++k) prod *= a[k];
                            acc += prod * dt[idx_dt(d, b, s, h)] * x[idx_x(d, b, s, h, p)] *
                                   Bm[idx_bc(d, b, s, g, n)];
                        }
                        final_state[idx_st(d, b, h, p, n)] = acc;
                    }
        }
    free(M); free(decay0); free(a);
    return 0;
}

/* ------------------------------------------------------------------------- */
/* Chunked form: the four stages, in fp64, with optional intermediates.      */
/*   l[b,h,c,i]   = sum_{k=cQ}^{cQ+i} dt_k A_h          (chunk-local, incl.)  */
/*   alpha[b,h,c] = exp(l[b,h,c,Q-1])                                         */
/*   w[b,h,c,i]   = exp(l[..,Q-1] - l[..,i]) * dt_{cQ+i}                      */
/*   S[b,c,h,p,n] = sum_i w_i x_i[p] B_i[n]                                   */
/*   sin[b,0,h]   = h0 ; sin[b,c+1,h] = alpha_c sin[b,c,h] + S[b,c,h]         */
/*   y_t[p]       = exp(l_t) sum_n C_t[n] sin[c][p,n]                         */
/*                + sum_{s<=t in chunk} exp(l_t - l_s) dt_s (C_t.B_s) x_s[p]  */
/*                + D_h x_t[p]                                                */
/* Intermediate pointers may be NULL.  sin has nc+1 entries per (b,h): entry */
/* nc is the final state.  Layouts: l, w [B,H,nc,Q]; alpha [B,H,nc];         */
/* S [B,nc,H,P,N]; sin [B,nc+1,H,P,N].                                        */
/* ------------------------------------------------------------------------- */
int oracle_ssd_chunked(const oracle_dims_t *d, int64_t Q, const double *x, const double *dt,
                       const double *A, const double *Bm, const double *Cm,
                       const double *D, const double *h0, double *y, double *final_state,
                       double *l_out, double *w_out, double *alpha_out, double *S_out,
                       double *sin_out) {
    if (!d || !x || !dt || !A || !Bm || !Cm || !y) return -1;
    if (d->ngroups <= 0 || d->nheads % d->ngroups != 0) return -2;
    if (Q <= 0 || d->seqlen % Q != 0) return -4;
    const int64_t T = d->seqlen, H = d->nheads, P = d->headdim, N = d->dstate;
    const int64_t nc = T / Q;
    double *l = (double *)malloc(sizeof(double) * Q);
    double *S = (double *)malloc(sizeof(double) * P * N);
    double *sin_c = (double *)malloc(sizeof(double) * P * N);
    if (!l || !S || !sin_c) {
        free(l); free(S); free(sin_c);
        return -3;
    }
    for (int64_t b = 0; b < d->batch; ++b)
        for (int64_t h = 0; h < H; ++h) {
            const int64_t g = group_of(d, h);
            for (int64_t i = 0; i < P * N; ++i) {
                const int64_t p = i / N, n = i % N;
                sin_c[i] = h0 ? h0[idx_st(d, b, h, p, n)] : 0.0;
            }
            for (int64_t c = 0; c < nc; ++c) {
                const int64_t t0 = c * Q;
                /* stage 1: chunk-local cumulative log-decay */
                double run = 0.0;
                for (int64_t i = 0; i < Q; ++i) {
                    run += dt[idx_dt(d, b, t0 + i, h)] * A[h];
                    l[i] = run;
                }
                const double alpha = exp(l[Q - 1]);
                if (l_out)
                    for (int64_t i = 0; i < Q; ++i) l_out[((b * H + h) * nc + c) * Q + i] = l[i];
                if (w_out)
                    for (int64_t i = 0; i < Q; ++i)
                        w_out[((b * H + h) * nc + c) * Q + i] =
                            exp(l[Q - 1] - l[i]) * dt[idx_dt(d, b, t0 + i, h)];
                if (alpha_out) alpha_out[(b * H + h) * nc + c] = alpha;
                /* stage 2: chunk state */
                for (int64_t p = 0; p < P; ++p)
                    for (int64_t n = 0; n < N; ++n) {
                        double acc = 0.0;
                        for (int64_t i = 0; i < Q; ++i) {
                            const double wi = exp(l[Q - 1] - l[i]) * dt[idx_dt(d, b, t0 + i, h)];
                            acc += wi * x[idx_x(d, b, t0 + i, h, p)] * Bm[idx_bc(d, b, t0 + i, g, n)];
                        }
                        S[p * N + n] = acc;
                    }
                if (S_out)
                    memcpy(S_out + (((b * nc + c) * H + h) * P * N), S, sizeof(double) * P * N);
                if (sin_out)
                    memcpy(sin_out + (((b * (nc + 1) + c) * H + h) * P * N), sin_c,
                           sizeof(double) * P * N);
                /* stage 4: outputs of this chunk from the incoming state */
                for (int64_t i = 0; i < Q; ++i) {
                    const int64_t t = t0 + i;
                    for (int64_t p = 0; p < P; ++p) {
                        double inter = 0.0;
                        for (int64_t n = 0; n < N; ++n)
                            inter += Cm[idx_bc(d, b, t, g, n)] * sin_c[p * N + n];
                        double intra = 0.0;
                        for (int64_t j = 0; j <= i; ++j) {
                            double cb = 0.0;
                            for (int64_t n = 0; n < N; ++n)
                                cb += Cm[idx_bc(d, b, t, g, n)] * Bm[idx_bc(d, b, t0 + j, g, n)];
                            intra += exp(l[i] - l[j]) * dt[idx_dt(d, b, t0 + j, h)] * cb *
                                     x[idx_x(d, b, t0 + j, h, p)];
                        }
                        y[idx_x(d, b, t, h, p)] =
                            exp(l[i]) * inter + intra + (D ? D[h] * x[idx_x(d, b, t, h, p)] : 0.0);
                    }
                }
                /* stage 3: hand the state to the next chunk */
                for (int64_t i = 0; i < P * N; ++i) sin_c[i] = alpha * sin_c[i] + S[i];
            }
            if (sin_out)
                memcpy(sin_out + (((b * (nc + 1) + nc) * H + h) * P * N), sin_c,
                       sizeof(double) * P * N);
            if (final_state)
                for (int64_t i = 0; i < P * N; ++i) {
                    const int64_t p = i / N, n = i % N;
                    final_state[idx_st(d, b, h, p, n)] = sin_c[i];
                }
        }
    free(l); free(S); free(sin_c);
    return 0;
}

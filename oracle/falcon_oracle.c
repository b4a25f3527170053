/*
 * falcon_oracle.c -- fp64 CPU oracle for the Falcon family of normalised
 * first-order fast-weight updates (Fast Weight Attention).
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, plain, obviously-correct
 * statement of what the GPU path computes.  Only the test-suite, the smoke
 * check and the CPU-baseline leg of the benchmark may load it.  It shares no
 * code, header, table or constant generator with the CUDA library.
 *
 * Sources (web pages on arXiv 2608.27763, cited by title and section):
 *   [EXPL]  "Fast Weight Attention：用于持续学习的快速权重注意力" (explainer),
 *           section 核心方法 (core method) 1-4.
 *   [SUMM]  "Fast Weight Attention for Continual Learning" (ai-feeds summary),
 *           section 方法 (method): 输入与状态定义 / 在线学习更新 / 计算形式与数值稳定.
 *   [NEWS]  "借鉴40年前的设想！字节Seed提出快速权重注意力推进大模型持续学习"
 *           (163.com article), section 02 Falcon (1) two objectives, (2) three
 *           granularities.
 *
 * Readings fixed where the pages are open (each one is also listed in the
 * design notes):
 *   R1  phi = L2 normalisation, phi(0) = 0 (identity exported for pins).
 *   R2  x_1 = 0 under the prefix pair (k_0 does not exist).
 *   R3  eta = beta / (eps + n) with n the squared input norm; eta = 0 when
 *       n = 0 (an empty sample writes nothing and forgets nothing).
 *   R4  positive decay alpha = max(1 - eta*lambda, 2^-20).
 *   R5  Falcon-2/2A: one step per value channel j (a row of S, S is d_v x d_k),
 *       sharing the normaliser eps + |x_t|^2.
 *   R6  Falcon-3/3A: window W_t = {max(1,t-Bw+1),...,t}; the Bw gradients are
 *       taken at S_{t-1}, summed, and scaled by one eta_t = beta_t/(eps+sum
 *       of |x_i|^2 over W_t) ("block normalisation").
 *   R7  read after write: o_t = S_t q_t, q used as given.
 *
 * Layouts (row-major, contiguous): q,k [B,H,L,dk]; v,out [B,H,L,dv];
 * beta [B,H,L] (variants 1,3,1A,3A) or [B,H,L,dv] (2,2A); lambda [H];
 * final_state [B,H,dv,dk].
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

enum { V_F1 = 0, V_F2 = 1, V_F3 = 2, V_F1A = 3, V_F2A = 4, V_F3A = 5 };
enum { FORM_RECURRENT = 0, FORM_MASKED = 1, FORM_CHUNK = 2 };
enum { PAIR_PREFIX = 0, PAIR_SAME_STEP = 1 };
enum { PHI_L2 = 0, PHI_IDENTITY = 1 };

#define ALPHA_FLOOR (1.0 / 1048576.0) /* 2^-20, reading R4 */

static int is_regression(int v) { return v == V_F1 || v == V_F2 || v == V_F3; }
static int is_per_channel(int v) { return v == V_F2 || v == V_F2A; }
static int is_window(int v) { return v == V_F3 || v == V_F3A; }

typedef struct {
    int variant, form, pairing, phi;
    int B, H, L, dk, dv, window, chunk;
    double eps;
    const double *q, *k, *v, *beta, *lambda;
    double *out, *final_state;
} job_t;

/* ------------------------------------------------------------------ */
/* Per-unit sample preparation: x_t, y_t, n_t, eta_t, alpha_t.          */
/* ------------------------------------------------------------------ */

typedef struct {
    int L, dk, dv, w, nch;   /* nch = dv for per-channel variants, else 1 */
    double *x;               /* [L][dk] samples x_t                        */
    const double *y;         /* [L][dv] targets y_t = v_t                  */
    const double *q;         /* [L][dk]                                    */
    double *eta;             /* [L][nch]                                   */
    double *alpha;           /* [L][nch]                                   */
} unit_t;

/* phi: [EXPL 核心方法 1] "projection of the previous key"; reading R1. */
static void apply_phi(int phi, const double *k, int dk, double *x)
{
    if (phi == PHI_IDENTITY) {
        for (int i = 0; i < dk; ++i) x[i] = k[i];
        return;
    }
    double s = 0.0;
    for (int i = 0; i < dk; ++i) s += k[i] * k[i];
    double nrm = sqrt(s);
    for (int i = 0; i < dk; ++i) x[i] = nrm > 0.0 ? k[i] / nrm : 0.0;
}

/*
 * Samples and step sizes for one (b,h) unit.
 *  x_t = phi(k_{t-1}) (prefix pair, [SUMM 输入与状态定义]; x_1 = 0 by R2) or
 *  x_t = phi(k_t) (same-step pair, [EXPL 核心方法 1] warning paragraph).
 *  eta_t = beta_t / (eps + n_t), the NLMS step [EXPL 核心方法 2, NLMS note],
 *  [NEWS 02 (1)]: "eta is the normalised step, beta the plasticity gain".
 *  alpha_t = 1 - eta_t*lambda, the L2-forgetting factor [NEWS 02 (1)].
 */
static void prepare_unit(const job_t *J, int b, int h, unit_t *u)
{
    const int L = J->L, dk = J->dk, dv = J->dv;
    const size_t bh = (size_t)b * J->H + h;
    const double *k = J->k + bh * (size_t)L * dk;
    u->L = L; u->dk = dk; u->dv = dv;
    u->w = is_window(J->variant) ? J->window : 1;
    u->nch = is_per_channel(J->variant) ? dv : 1;
    u->y = J->v + bh * (size_t)L * dv;
    u->q = J->q + bh * (size_t)L * dk;
    u->x = (double *)calloc((size_t)L * dk, sizeof(double));
    u->eta = (double *)calloc((size_t)L * u->nch, sizeof(double));
    u->alpha = (double *)calloc((size_t)L * u->nch, sizeof(double));

    for (int t = 0; t < L; ++t) {
        double *xt = u->x + (size_t)t * dk;
        if (J->pairing == PAIR_SAME_STEP)
            apply_phi(J->phi, k + (size_t)t * dk, dk, xt);
        else if (t == 0)
            memset(xt, 0, sizeof(double) * dk);
        else
            apply_phi(J->phi, k + (size_t)(t - 1) * dk, dk, xt);
    }
    const double lam = J->lambda[h];
    const double *beta = J->beta + bh * (size_t)L * u->nch;
    for (int t = 0; t < L; ++t) {
        /* normaliser: |x_t|^2, or the window's energy for Falcon-3/3A (R6) */
        double n = 0.0;
        int i0 = t - u->w + 1;
        if (i0 < 0) i0 = 0;
        for (int i = i0; i <= t; ++i)
            for (int c = 0; c < dk; ++c) n += u->x[(size_t)i * dk + c] * u->x[(size_t)i * dk + c];
        for (int j = 0; j < u->nch; ++j) {
            double eta = n > 0.0 ? beta[(size_t)t * u->nch + j] / (J->eps + n) : 0.0;
            double a = 1.0 - eta * lam;
            if (a < ALPHA_FLOOR) a = ALPHA_FLOOR;
            u->eta[(size_t)t * u->nch + j] = eta;
            u->alpha[(size_t)t * u->nch + j] = a;
        }
    }
}

static void free_unit(unit_t *u)
{
    free(u->x); free(u->eta); free(u->alpha);
}

static double dot(const double *a, const double *b, int n)
{
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* ------------------------------------------------------------------ */
/* Form 1: recurrent -- the definition.                                 */
/* ------------------------------------------------------------------ */

/*
 * S_t = S_{t-1} - eta_t grad L(S_{t-1}; x_t, y_t) plus L2 forgetting
 * [EXPL 核心方法 1], [NEWS 02 (1)]:
 *   regression     grad = (S x - y) x^T  ->  S_t = alpha S_{t-1} + eta (y - S_{t-1} x) x^T
 *   inner product  grad = -y x^T         ->  S_t = alpha S_{t-1} + eta y x^T
 * Falcon-2/2A take eta, alpha per value channel (row j of S) [NEWS 02 (2)];
 * Falcon-3/3A sum the gradients of the last Bw samples, all at S_{t-1}
 * [EXPL 核心方法 2 table], [NEWS 02 (2)].  Output o_t = S_t q_t (R7).
 */
static void unit_recurrent(const job_t *J, const unit_t *u, double *out, double *S)
{
    const int L = u->L, dk = u->dk, dv = u->dv, w = u->w;
    double *res = (double *)calloc((size_t)w * dv, sizeof(double));
    memset(S, 0, sizeof(double) * (size_t)dv * dk);
    for (int t = 0; t < L; ++t) {
        int i0 = t - w + 1;
        if (i0 < 0) i0 = 0;
        /* residuals (or targets) at S_{t-1} for every sample of the window */
        for (int i = i0; i <= t; ++i) {
            const double *xi = u->x + (size_t)i * dk;
            const double *yi = u->y + (size_t)i * dv;
            for (int j = 0; j < dv; ++j)
                res[(size_t)(i - i0) * dv + j] =
                    is_regression(J->variant) ? yi[j] - dot(S + (size_t)j * dk, xi, dk) : yi[j];
        }
        for (int j = 0; j < dv; ++j) {
            const int ch = u->nch > 1 ? j : 0;
            const double eta = u->eta[(size_t)t * u->nch + ch];
            const double a = u->alpha[(size_t)t * u->nch + ch];
            double *Sj = S + (size_t)j * dk;
            for (int c = 0; c < dk; ++c) {
                double g = 0.0;
                for (int i = i0; i <= t; ++i) g += res[(size_t)(i - i0) * dv + j] * u->x[(size_t)i * dk + c];
                Sj[c] = a * Sj[c] + eta * g;
            }
        }
        const double *qt = u->q + (size_t)t * dk;
        for (int j = 0; j < dv; ++j) out[(size_t)t * dv + j] = dot(S + (size_t)j * dk, qt, dk);
    }
    free(res);
}

/* ------------------------------------------------------------------ */
/* Forms 2 and 3: masked-parallel and chunk-parallel.                   */
/* ------------------------------------------------------------------ */

/*
 * Both forms unroll the recurrence over a span [c0,c1) of positions that
 * starts from a carried state S0 ([EXPL 核心方法 3], [SUMM 计算形式与数值稳定],
 * [NEWS 02 (2)] "chunks are parallel inside and pass only a fixed-size state
 * between them").  The masked-parallel form is one span covering the whole
 * sequence with S0 = 0; the chunk-parallel form is a sequence of spans of
 * length `chunk` that hand S0 on.
 *
 * With G_t = sum_{c0<=r<=t} log alpha_r (per channel for Falcon-2/2A) and
 * G_{c0-1} = 0, the state inside the span is
 *   S_t = e^{G_t} S0 + sum_{c0<=s<=t} e^{G_t-G_s} eta_s sum_{i in W_s} r_{s,i} x_i^T,
 * where r_{s,i} = y_i - S_{s-1} x_i for the regression family and y_i for
 * the inner-product family (W_s = {s} outside Falcon-3/3A).  Substituting
 * S_{t-1} into r_{t,i} gives the causal (lower-triangular, unit-diagonal)
 * system solved below by forward substitution, channel by channel:
 *   r_{t,i} = y_i - e^{G_{t-1}} S0 x_i
 *             - sum_{c0<=s<t} e^{G_{t-1}-G_s} eta_s sum_{i' in W_s} (x_i'.x_i) r_{s,i'}.
 * The outputs are o_t = S_t q_t with S_t as above, and the span ends with
 * S0 <- S_{c1-1}.
 */
static void unit_span(const job_t *J, const unit_t *u, int c0, int c1, double *S0, double *out)
{
    const int dk = u->dk, dv = u->dv, w = u->w, n = c1 - c0;
    const int reg = is_regression(J->variant);
    double *G = (double *)malloc(sizeof(double) * (size_t)n);
    double *r = (double *)malloc(sizeof(double) * (size_t)n * w); /* r[(t-c0)*w + m], i = t-w+1+m */
    double *Snew = (double *)malloc(sizeof(double) * (size_t)dk);

    for (int j = 0; j < dv; ++j) {
        const int ch = u->nch > 1 ? j : 0;
        const double *S0j = S0 + (size_t)j * dk;
        double acc = 0.0;
        for (int t = c0; t < c1; ++t) {
            acc += log(u->alpha[(size_t)t * u->nch + ch]);
            G[t - c0] = acc;
        }
        /* unknowns, in causal order */
        for (int t = c0; t < c1; ++t) {
            const double Gtm1 = t > c0 ? G[t - 1 - c0] : 0.0;
            for (int m = 0; m < w; ++m) {
                const int i = t - w + 1 + m;
                double val = 0.0;
                if (i >= 0) {
                    const double *xi = u->x + (size_t)i * dk;
                    val = u->y[(size_t)i * dv + j];
                    if (reg) {
                        val -= exp(Gtm1) * dot(S0j, xi, dk);
                        for (int s = c0; s < t; ++s) {
                            const double coef = exp(Gtm1 - G[s - c0]) * u->eta[(size_t)s * u->nch + ch];
                            for (int m2 = 0; m2 < w; ++m2) {
                                const int i2 = s - w + 1 + m2;
                                if (i2 < 0) continue;
                                val -= coef * dot(u->x + (size_t)i2 * dk, xi, dk) * r[(size_t)(s - c0) * w + m2];
                            }
                        }
                    }
                }
                r[(size_t)(t - c0) * w + m] = val;
            }
        }
        /* outputs o_t = S_t q_t */
        for (int t = c0; t < c1; ++t) {
            const double *qt = u->q + (size_t)t * dk;
            double o = exp(G[t - c0]) * dot(S0j, qt, dk);
            for (int s = c0; s <= t; ++s) {
                const double coef = exp(G[t - c0] - G[s - c0]) * u->eta[(size_t)s * u->nch + ch];
                for (int m = 0; m < w; ++m) {
                    const int i = s - w + 1 + m;
                    if (i < 0) continue;
                    o += coef * dot(u->x + (size_t)i * dk, qt, dk) * r[(size_t)(s - c0) * w + m];
                }
            }
            out[(size_t)t * dv + j] = o;
        }
        /* carried state S0 <- S_{c1-1} */
        const double Gend = G[n - 1];
        for (int c = 0; c < dk; ++c) Snew[c] = exp(Gend) * S0j[c];
        for (int s = c0; s < c1; ++s) {
            const double coef = exp(Gend - G[s - c0]) * u->eta[(size_t)s * u->nch + ch];
            for (int m = 0; m < w; ++m) {
                const int i = s - w + 1 + m;
                if (i < 0) continue;
                const double *xi = u->x + (size_t)i * dk;
                for (int c = 0; c < dk; ++c) Snew[c] += coef * r[(size_t)(s - c0) * w + m] * xi[c];
            }
        }
        memcpy(S0 + (size_t)j * dk, Snew, sizeof(double) * dk);
    }
    free(G); free(r); free(Snew);
}

static void unit_run(const job_t *J, int b, int h)
{
    unit_t u;
    prepare_unit(J, b, h, &u);
    const size_t bh = (size_t)b * J->H + h;
    double *out = J->out + bh * (size_t)J->L * J->dv;
    double *S = (double *)calloc((size_t)J->dv * J->dk, sizeof(double));
    if (J->L > 0) {
        if (J->form == FORM_RECURRENT) {
            unit_recurrent(J, &u, out, S);
        } else {
            const int span = J->form == FORM_MASKED ? J->L : J->chunk;
            for (int c0 = 0; c0 < J->L; c0 += span) {
                int c1 = c0 + span;
                if (c1 > J->L) c1 = J->L;
                unit_span(J, &u, c0, c1, S, out);
            }
        }
    }
    if (J->final_state)
        memcpy(J->final_state + bh * (size_t)J->dv * J->dk, S, sizeof(double) * (size_t)J->dv * J->dk);
    free(S);
    free_unit(&u);
}

/* ------------------------------------------------------------------ */
/* Threading over independent (b,h) units.                             */
/* ------------------------------------------------------------------ */

typedef struct {
    const job_t *J;
    int tid, nthreads;
} worker_t;

static void *worker(void *arg)
{
    const worker_t *W = (const worker_t *)arg;
    const int units = W->J->B * W->J->H;
    for (int n = W->tid; n < units; n += W->nthreads) unit_run(W->J, n / W->J->H, n % W->J->H);
    return NULL;
}

static int run_threads(const job_t *J, int nthreads)
{
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    const int units = J->B * J->H;
    if (nthreads > units) nthreads = units > 0 ? units : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    worker_t *ws = (worker_t *)malloc(sizeof(worker_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) {
        ws[i].J = J; ws[i].tid = i; ws[i].nthreads = nthreads;
        pthread_create(&th[i], NULL, worker, &ws[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th); free(ws);
    return nthreads;
}

/* Returns the number of threads used (>0) or a negative error. */
int oracle_fwd(int variant, int form, int pairing, int phi,
               const double *q, const double *k, const double *v, const double *beta,
               const double *lambda, double eps, int window, int B, int H, int L, int dk, int dv,
               int chunk, double *out, double *final_state, int nthreads)
{
    if (variant < 0 || variant > 5 || form < 0 || form > 2) return -2;
    if (B < 0 || H < 0 || L < 0 || dk <= 0 || dv <= 0) return -3;
    if (form == FORM_CHUNK && chunk <= 0) return -4;
    if (is_window(variant) && window < 1) return -6;
    job_t J = {variant, form, pairing, phi, B, H, L, dk, dv, window, chunk, eps,
               q, k, v, beta, lambda, out, final_state};
    return run_threads(&J, nthreads);
}

/* ------------------------------------------------------------------ */
/* Recurrent form continuing an earlier segment (initial state + carry). */
/* ------------------------------------------------------------------ */

/*
 * A segment that continues a sequence: the state starts at S0 (zeros when
 * NULL) and the samples before the segment are the decode carry (the same
 * layout as oracle_decode_step): x_prev = phi(k) of the token before the
 * segment, which is x_1 of the segment under the prefix pair, and for
 * Falcon-3/3A the Bw-1 samples before it, win[m] = (x, y), oldest first.
 * NULL carries are zeros, which is exactly the start of a sequence (R2: an
 * all-zero sample adds no energy and no gradient).  The definition is the
 * recurrent form above, run over the carried samples followed by the
 * segment's.  Under the same-step pair ([EXPL 核心方法 1] warning paragraph)
 * the segment's samples are (phi(k_t), v_t), so x_prev is not read, and the
 * window carry holds the same-step samples before the segment.
 */
typedef struct {
    int variant, pairing, phi, B, H, L, dk, dv, w;
    double eps;
    const double *q, *k, *v, *beta, *lambda, *S0, *x_prev, *win;
    double *out, *final_state;
} carry_job_t;

static void carry_unit_run(const carry_job_t *C, int b, int h)
{
    const int L = C->L, dk = C->dk, dv = C->dv, w = C->w, P = w - 1;
    const int nch = is_per_channel(C->variant) ? dv : 1;
    const size_t bh = (size_t)b * C->H + h;
    const double *k = C->k + bh * (size_t)L * dk, *v = C->v + bh * (size_t)L * dv;
    const double *q = C->q + bh * (size_t)L * dk, *beta = C->beta + bh * (size_t)L * nch;
    /* samples at positions -P .. L-1 (index i + P) */
    double *X = (double *)calloc((size_t)(L + P) * dk, sizeof(double));
    double *Y = (double *)calloc((size_t)(L + P) * dv, sizeof(double));
    for (int m = 0; m < P && C->win; ++m) {
        const double *wm = C->win + (bh * (size_t)P + m) * (size_t)(dk + dv);
        memcpy(X + (size_t)m * dk, wm, sizeof(double) * dk);
        memcpy(Y + (size_t)m * dv, wm + dk, sizeof(double) * dv);
    }
    for (int t = 0; t < L; ++t) {
        double *xt = X + (size_t)(t + P) * dk;
        if (C->pairing == PAIR_SAME_STEP) {
            apply_phi(C->phi, k + (size_t)t * dk, dk, xt); /* the segment's own key */
        } else if (t == 0) {
            if (C->x_prev) memcpy(xt, C->x_prev + bh * (size_t)dk, sizeof(double) * dk);
        } else {
            apply_phi(C->phi, k + (size_t)(t - 1) * dk, dk, xt);
        }
        memcpy(Y + (size_t)(t + P) * dv, v + (size_t)t * dv, sizeof(double) * dv);
    }
    double *S = (double *)calloc((size_t)dv * dk, sizeof(double));
    if (C->S0) memcpy(S, C->S0 + bh * (size_t)dv * dk, sizeof(double) * (size_t)dv * dk);
    double *res = (double *)calloc((size_t)w * dv, sizeof(double));
    double *out = C->out + bh * (size_t)L * dv;
    const double lam = C->lambda[h];
    for (int t = 0; t < L; ++t) {
        /* window t-w+1 .. t, all present among the carried samples */
        double n = 0.0;
        for (int i = t - w + 1; i <= t; ++i) n += dot(X + (size_t)(i + P) * dk, X + (size_t)(i + P) * dk, dk);
        for (int i = t - w + 1; i <= t; ++i) {
            const double *xi = X + (size_t)(i + P) * dk, *yi = Y + (size_t)(i + P) * dv;
            for (int j = 0; j < dv; ++j)
                res[(size_t)(i - (t - w + 1)) * dv + j] =
                    is_regression(C->variant) ? yi[j] - dot(S + (size_t)j * dk, xi, dk) : yi[j];
        }
        for (int j = 0; j < dv; ++j) {
            const int ch = nch > 1 ? j : 0;
            const double eta = n > 0.0 ? beta[(size_t)t * nch + ch] / (C->eps + n) : 0.0;
            double a = 1.0 - eta * lam;
            if (a < ALPHA_FLOOR) a = ALPHA_FLOOR;
            double *Sj = S + (size_t)j * dk;
            for (int c = 0; c < dk; ++c) {
                double g = 0.0;
                for (int i = t - w + 1; i <= t; ++i)
                    g += res[(size_t)(i - (t - w + 1)) * dv + j] * X[(size_t)(i + P) * dk + c];
                Sj[c] = a * Sj[c] + eta * g;
            }
        }
        for (int j = 0; j < dv; ++j) out[(size_t)t * dv + j] = dot(S + (size_t)j * dk, q + (size_t)t * dk, dk);
    }
    if (C->final_state) memcpy(C->final_state + bh * (size_t)dv * dk, S, sizeof(double) * (size_t)dv * dk);
    free(X); free(Y); free(S); free(res);
}

typedef struct {
    const carry_job_t *C;
    int tid, nthreads;
} carry_worker_t;

static void *carry_worker(void *arg)
{
    const carry_worker_t *W = (const carry_worker_t *)arg;
    const int units = W->C->B * W->C->H;
    for (int n = W->tid; n < units; n += W->nthreads) carry_unit_run(W->C, n / W->C->H, n % W->C->H);
    return NULL;
}

/* Returns the number of threads used (>0) or a negative error. */
int oracle_fwd_carry(int variant, int pairing, int phi, const double *q, const double *k, const double *v,
                     const double *beta, const double *lambda, double eps, int window, int B, int H, int L, int dk,
                     int dv, const double *S0, const double *x_prev, const double *win,
                     double *out, double *final_state, int nthreads)
{
    if (variant < 0 || variant > 5 || pairing < 0 || pairing > 1) return -2;
    if (B < 0 || H < 0 || L < 0 || dk <= 0 || dv <= 0) return -3;
    if (is_window(variant) && window < 1) return -6;
    carry_job_t C = {variant, pairing, phi, B, H, L, dk, dv, is_window(variant) ? window : 1, eps,
                     q, k, v, beta, lambda, S0, x_prev, win, out, final_state};
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    const int units = B * H;
    if (nthreads > units) nthreads = units > 0 ? units : 1;
    if (nthreads < 1) nthreads = 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    carry_worker_t *ws = (carry_worker_t *)malloc(sizeof(carry_worker_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) {
        ws[i].C = &C; ws[i].tid = i; ws[i].nthreads = nthreads;
        pthread_create(&th[i], NULL, carry_worker, &ws[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th); free(ws);
    return nthreads;
}

/* ------------------------------------------------------------------ */
/* Single-token recurrent step with its carry (decode).                 */
/* ------------------------------------------------------------------ */

/*
 * One recurrent step per (n,h), [EXPL 核心方法 3] "recurrent: O(d^2) per
 * step, for inference".  Carry: x_prev = phi(k_{t-1}) (zeros before the first
 * token, R2) and, for Falcon-3/3A, the previous Bw-1 samples win[m] =
 * (x, y), oldest first (zeros where the sequence had fewer samples, which
 * contribute nothing: an all-zero x adds no energy and no gradient).
 * Under the same-step pair ([EXPL 核心方法 1] warning paragraph) the step's
 * sample is (phi(k_t), v_t) and x_prev is not read (it may be NULL; when
 * given it is still set to phi(k_t)).
 * Layouts: state [N,H,dv,dk]; x_prev [N,H,dk]; win [N,H,Bw-1,dk+dv];
 * q,k [N,H,dk]; v,out [N,H,dv]; beta [N,H] or [N,H,dv].
 */
int oracle_decode_step(int variant, int pairing, int phi, const double *q, const double *k, const double *v,
                       const double *beta, const double *lambda, double eps, int window,
                       int N, int H, int dk, int dv, double *state, double *x_prev, double *win,
                       double *out)
{
    if (variant < 0 || variant > 5 || pairing < 0 || pairing > 1) return -2;
    if (pairing == PAIR_PREFIX && !x_prev) return -1;
    const int w = is_window(variant) ? window : 1;
    if (w < 1) return -6;
    const int nch = is_per_channel(variant) ? dv : 1;
    double *xs = (double *)malloc(sizeof(double) * (size_t)w * dk);
    double *ys = (double *)malloc(sizeof(double) * (size_t)w * dv);
    double *res = (double *)malloc(sizeof(double) * (size_t)w * dv);
    for (int nh = 0; nh < N * H; ++nh) {
        const int h = nh % H;
        double *S = state + (size_t)nh * dv * dk;
        /* window samples, oldest first; the current one is (x_prev, v_t) */
        for (int m = 0; m < w - 1; ++m) {
            const double *slot = win + ((size_t)nh * (w - 1) + m) * (dk + dv);
            memcpy(xs + (size_t)m * dk, slot, sizeof(double) * dk);
            memcpy(ys + (size_t)m * dv, slot + dk, sizeof(double) * dv);
        }
        if (pairing == PAIR_SAME_STEP)
            apply_phi(phi, k + (size_t)nh * dk, dk, xs + (size_t)(w - 1) * dk);
        else
            memcpy(xs + (size_t)(w - 1) * dk, x_prev + (size_t)nh * dk, sizeof(double) * dk);
        memcpy(ys + (size_t)(w - 1) * dv, v + (size_t)nh * dv, sizeof(double) * dv);
        double n = 0.0;
        for (int m = 0; m < w; ++m) n += dot(xs + (size_t)m * dk, xs + (size_t)m * dk, dk);
        for (int m = 0; m < w; ++m)
            for (int j = 0; j < dv; ++j)
                res[(size_t)m * dv + j] = is_regression(variant)
                                              ? ys[(size_t)m * dv + j] - dot(S + (size_t)j * dk, xs + (size_t)m * dk, dk)
                                              : ys[(size_t)m * dv + j];
        for (int j = 0; j < dv; ++j) {
            const double bt = beta[(size_t)nh * nch + (nch > 1 ? j : 0)];
            const double eta = n > 0.0 ? bt / (eps + n) : 0.0;
            double a = 1.0 - eta * lambda[h];
            if (a < ALPHA_FLOOR) a = ALPHA_FLOOR;
            double *Sj = S + (size_t)j * dk;
            for (int c = 0; c < dk; ++c) {
                double g = 0.0;
                for (int m = 0; m < w; ++m) g += res[(size_t)m * dv + j] * xs[(size_t)m * dk + c];
                Sj[c] = a * Sj[c] + eta * g;
            }
            out[(size_t)nh * dv + j] = dot(Sj, q + (size_t)nh * dk, dk);
        }
        /* shift the carry: drop the oldest sample, append the current one */
        for (int m = 0; m + 1 < w - 1; ++m)
            memcpy(win + ((size_t)nh * (w - 1) + m) * (dk + dv),
                   win + ((size_t)nh * (w - 1) + m + 1) * (dk + dv), sizeof(double) * (dk + dv));
        if (w > 1) {
            double *slot = win + ((size_t)nh * (w - 1) + (w - 2)) * (dk + dv);
            memcpy(slot, xs + (size_t)(w - 1) * dk, sizeof(double) * dk);
            memcpy(slot + dk, ys + (size_t)(w - 1) * dv, sizeof(double) * dv);
        }
        if (x_prev) apply_phi(phi, k + (size_t)nh * dk, dk, x_prev + (size_t)nh * dk);
    }
    free(xs); free(ys); free(res);
    return 0;
}

/*
 * Decode carry after a prefill of L tokens: x_prev = phi(k_L) and the window
 * holds the samples (x_i, y_i) for i = L-Bw+2..L, oldest first, zeros for
 * i < 1; x_i = phi(k_{i-1}) under the prefix pair, phi(k_i) under the
 * same-step pair.
 */
int oracle_carry_from_prefill(int variant, int pairing, int phi, const double *k, const double *v, int window,
                              int B, int H, int L, int dk, int dv, double *x_prev, double *win)
{
    const int w = is_window(variant) ? window : 1;
    if (w < 1) return -6;
    if (pairing < 0 || pairing > 1) return -2;
    for (int bh = 0; bh < B * H; ++bh) {
        const double *kb = k + (size_t)bh * L * dk;
        const double *vb = v + (size_t)bh * L * dv;
        if (L > 0) apply_phi(phi, kb + (size_t)(L - 1) * dk, dk, x_prev + (size_t)bh * dk);
        else memset(x_prev + (size_t)bh * dk, 0, sizeof(double) * dk);
        for (int m = 0; m < w - 1; ++m) {
            double *slot = win + ((size_t)bh * (w - 1) + m) * (dk + dv);
            const int i = L - (w - 1) + m; /* 0-based sample index */
            memset(slot, 0, sizeof(double) * (dk + dv));
            if (i < 0) continue;
            if (pairing == PAIR_SAME_STEP) apply_phi(phi, kb + (size_t)i * dk, dk, slot);
            else if (i >= 1) apply_phi(phi, kb + (size_t)(i - 1) * dk, dk, slot);
            memcpy(slot + dk, vb + (size_t)i * dv, sizeof(double) * dv);
        }
    }
    return 0;
}

/* ------------------------------------------------------------------ */
/* Reverse mode of the recurrent definition (the backward pass).        */
/* ------------------------------------------------------------------ */

/*
 * Gradients of a scalar loss L through the recurrent form, given dL/do_t
 * (dout [B,H,L,dv]) and dL/dS_L (dstate [B,H,dv,dk], NULL for zero), for
 * every variant, pairing and feature map, from S_0 = 0 (no carry).  The
 * chunk form trains on the same function ([EXPL 核心方法 3], [NEWS 02 (2)]);
 * this is its derivative taken step by step, latest step first:
 *   o_t = S_t q_t                      dq_t = S_t^T do_t,   Gs += do_t q_t^T
 *   S_t = alpha_t S_{t-1} + eta_t U_t  dalpha_t += <Gs, S_{t-1}>, deta_t += <Gs, U_t>
 *   U_t = sum_{i in W_t} e_{t,i} x_i^T, e_{t,i} = y_i - S_{t-1} x_i (regression) or y_i
 *                                      de_{t,i} = eta_t Gs x_i,  dx_i += eta_t Gs^T e_{t,i}
 *                                      regression: dy_i += de, dx_i -= S_{t-1}^T de,
 *                                                  Gs <- alpha_t Gs - sum_i de x_i^T
 *                                      inner product: dy_i += de, Gs <- alpha_t Gs
 * (row j with its own eta, alpha for Falcon-2/2A; the inner products above
 * then stay within the row).  Then the steps (R3, R4):
 *   alpha = max(1 - eta lambda, 2^-20): deta += -lambda dalpha, dlambda += -eta dalpha
 *     where 1 - eta lambda > 2^-20; no gradient where the floor holds;
 *   eta = beta / (eps + n) (0 when n = 0): dbeta = deta / (eps + n), dn += -deta beta / (eps + n)^2;
 *   n = sum_{i in W_t} |x_i|^2: dx_i += 2 dn x_i;
 *   x = k / |k| (R1): dk = (dx - x (x . dx)) / |k|, 0 at k = 0; identity: dk = dx.
 * Outputs (all [B,H,...] like the inputs): dq, dk, dv, dbeta and dlambda [H]
 * (summed over b).  The state history is kept whole: meant for small cases.
 */
typedef struct {
    int variant, pairing, phi, B, H, L, dk, dv, w;
    double eps;
    const double *q, *k, *v, *beta, *lambda, *dout, *dstate;
    double *dq, *dkk, *dvv, *dbeta, *dlam_bh;  /* dlam_bh [B*H], summed by the caller */
    double *dlam_l1_bh;                        /* [B*H]: sum of |eta_t dL/dalpha_t| over the dlambda terms */
} bwd_job_t;

static void bwd_unit_run(const bwd_job_t *Bj, int b, int h)
{
    const int L = Bj->L, dk = Bj->dk, dv = Bj->dv, w = Bj->w;
    const size_t bh = (size_t)b * Bj->H + h;
    job_t J = {Bj->variant, FORM_RECURRENT, Bj->pairing, Bj->phi, Bj->B, Bj->H, L, dk, dv, w, 1, Bj->eps,
               Bj->q, Bj->k, Bj->v, Bj->beta, Bj->lambda, NULL, NULL};
    unit_t u;
    prepare_unit(&J, b, h, &u);
    const int nch = u.nch, reg = is_regression(Bj->variant);
    const size_t SS = (size_t)dv * dk;
    /* forward: the whole history S_0 .. S_L (S_0 = 0) */
    double *hist = (double *)calloc((size_t)(L + 1) * SS, sizeof(double));
    double *res = (double *)calloc((size_t)w * dv, sizeof(double));
    for (int t = 0; t < L; ++t) {
        const double *Sp = hist + (size_t)t * SS;
        double *Sn = hist + (size_t)(t + 1) * SS;
        int i0 = t - w + 1;
        if (i0 < 0) i0 = 0;
        for (int i = i0; i <= t; ++i)
            for (int j = 0; j < dv; ++j)
                res[(size_t)(i - i0) * dv + j] = reg ? u.y[(size_t)i * dv + j] - dot(Sp + (size_t)j * dk, u.x + (size_t)i * dk, dk)
                                                     : u.y[(size_t)i * dv + j];
        for (int j = 0; j < dv; ++j) {
            const int ch = nch > 1 ? j : 0;
            const double eta = u.eta[(size_t)t * nch + ch], a = u.alpha[(size_t)t * nch + ch];
            for (int c = 0; c < dk; ++c) {
                double g = 0.0;
                for (int i = i0; i <= t; ++i) g += res[(size_t)(i - i0) * dv + j] * u.x[(size_t)i * dk + c];
                Sn[(size_t)j * dk + c] = a * Sp[(size_t)j * dk + c] + eta * g;
            }
        }
    }
    /* backward */
    double *Gs = (double *)calloc(SS, sizeof(double));
    double *Gn = (double *)calloc(SS, sizeof(double));
    double *dx = (double *)calloc((size_t)L * dk, sizeof(double));
    double *deta = (double *)calloc((size_t)L * nch, sizeof(double));
    double *dalpha = (double *)calloc((size_t)L * nch, sizeof(double));
    double *de = (double *)calloc((size_t)w * dv, sizeof(double));
    double *dq = Bj->dq + bh * (size_t)L * dk;
    double *dvv = Bj->dvv + bh * (size_t)L * dv;
    memset(dvv, 0, sizeof(double) * (size_t)L * dv);
    if (Bj->dstate) memcpy(Gs, Bj->dstate + bh * SS, sizeof(double) * SS);
    const double *dout = Bj->dout + bh * (size_t)L * dv;
    for (int t = L - 1; t >= 0; --t) {
        const double *St = hist + (size_t)(t + 1) * SS, *Sp = hist + (size_t)t * SS;
        const double *qt = u.q + (size_t)t * dk, *dot_ = dout + (size_t)t * dv;
        for (int c = 0; c < dk; ++c) {
            double s = 0.0;
            for (int j = 0; j < dv; ++j) s += St[(size_t)j * dk + c] * dot_[j];
            dq[(size_t)t * dk + c] = s;
        }
        for (int j = 0; j < dv; ++j)
            for (int c = 0; c < dk; ++c) Gs[(size_t)j * dk + c] += dot_[j] * qt[c];
        int i0 = t - w + 1;
        if (i0 < 0) i0 = 0;
        for (int i = i0; i <= t; ++i)
            for (int j = 0; j < dv; ++j)
                res[(size_t)(i - i0) * dv + j] = reg ? u.y[(size_t)i * dv + j] - dot(Sp + (size_t)j * dk, u.x + (size_t)i * dk, dk)
                                                     : u.y[(size_t)i * dv + j];
        for (int j = 0; j < dv; ++j) {
            const int ch = nch > 1 ? j : 0;
            const double eta = u.eta[(size_t)t * nch + ch];
            const double *Gj = Gs + (size_t)j * dk, *Spj = Sp + (size_t)j * dk;
            dalpha[(size_t)t * nch + ch] += dot(Gj, Spj, dk);
            for (int i = i0; i <= t; ++i) {
                const double *xi = u.x + (size_t)i * dk;
                const double e = res[(size_t)(i - i0) * dv + j];
                const double gx = dot(Gj, xi, dk);
                deta[(size_t)t * nch + ch] += e * gx;
                de[(size_t)(i - i0) * dv + j] = eta * gx;
                for (int c = 0; c < dk; ++c) dx[(size_t)i * dk + c] += eta * Gj[c] * e;
            }
        }
        for (int i = i0; i <= t; ++i) {
            for (int j = 0; j < dv; ++j) {
                const double d = de[(size_t)(i - i0) * dv + j];
                dvv[(size_t)i * dv + j] += d;
                if (reg)
                    for (int c = 0; c < dk; ++c) dx[(size_t)i * dk + c] -= Sp[(size_t)j * dk + c] * d;
            }
        }
        /* dL/dS_{t-1} */
        for (int j = 0; j < dv; ++j) {
            const int ch = nch > 1 ? j : 0;
            const double a = u.alpha[(size_t)t * nch + ch];
            for (int c = 0; c < dk; ++c) {
                double g = a * Gs[(size_t)j * dk + c];
                if (reg)
                    for (int i = i0; i <= t; ++i) g -= de[(size_t)(i - i0) * dv + j] * u.x[(size_t)i * dk + c];
                Gn[(size_t)j * dk + c] = g;
            }
        }
        memcpy(Gs, Gn, sizeof(double) * SS);
    }
    /* the steps, the normaliser, the feature map */
    const double lam = Bj->lambda[h];
    const double *beta = Bj->beta + bh * (size_t)L * nch;
    double *dbeta = Bj->dbeta + bh * (size_t)L * nch;
    double dlam = 0.0, dlam_l1 = 0.0;
    for (int t = 0; t < L; ++t) {
        int i0 = t - w + 1;
        if (i0 < 0) i0 = 0;
        double n = 0.0;
        for (int i = i0; i <= t; ++i) n += dot(u.x + (size_t)i * dk, u.x + (size_t)i * dk, dk);
        double dn = 0.0;
        for (int ch = 0; ch < nch; ++ch) {
            const double eta = u.eta[(size_t)t * nch + ch];
            double de_ = deta[(size_t)t * nch + ch];
            if (1.0 - eta * lam > ALPHA_FLOOR) {
                de_ += -lam * dalpha[(size_t)t * nch + ch];
                dlam += -eta * dalpha[(size_t)t * nch + ch];
                dlam_l1 += fabs(eta * dalpha[(size_t)t * nch + ch]);
            }
            if (n > 0.0) {
                const double bt = beta[(size_t)t * nch + ch];
                dbeta[(size_t)t * nch + ch] = de_ / (Bj->eps + n);
                dn += -de_ * bt / ((Bj->eps + n) * (Bj->eps + n));
            } else {
                dbeta[(size_t)t * nch + ch] = 0.0;
            }
        }
        for (int i = i0; i <= t; ++i)
            for (int c = 0; c < dk; ++c) dx[(size_t)i * dk + c] += 2.0 * dn * u.x[(size_t)i * dk + c];
    }
    double *dkk = Bj->dkk + bh * (size_t)L * dk;
    memset(dkk, 0, sizeof(double) * (size_t)L * dk);
    const double *kk = Bj->k + bh * (size_t)L * dk;
    for (int i = 0; i < L; ++i) {
        const int kr = Bj->pairing == PAIR_SAME_STEP ? i : i - 1;  /* x_i = phi(k_kr); x_0 = 0 under the prefix pair */
        if (kr < 0) continue;
        const double *xi = u.x + (size_t)i * dk, *dxi = dx + (size_t)i * dk, *ki = kk + (size_t)kr * dk;
        if (Bj->phi == PHI_IDENTITY) {
            for (int c = 0; c < dk; ++c) dkk[(size_t)kr * dk + c] += dxi[c];
        } else {
            const double nrm = sqrt(dot(ki, ki, dk));
            if (nrm > 0.0) {
                const double xd = dot(xi, dxi, dk);
                for (int c = 0; c < dk; ++c) dkk[(size_t)kr * dk + c] += (dxi[c] - xi[c] * xd) / nrm;
            }
        }
    }
    Bj->dlam_bh[bh] = dlam;
    Bj->dlam_l1_bh[bh] = dlam_l1;
    free(hist); free(res); free(Gs); free(Gn); free(dx); free(deta); free(dalpha); free(de);
    free_unit(&u);
}

typedef struct {
    const bwd_job_t *J;
    int tid, nthreads;
} bwd_worker_t;

static void *bwd_worker(void *arg)
{
    const bwd_worker_t *W = (const bwd_worker_t *)arg;
    const int units = W->J->B * W->J->H;
    for (int n = W->tid; n < units; n += W->nthreads) bwd_unit_run(W->J, n / W->J->H, n % W->J->H);
    return NULL;
}

/* dlambda_l1 (optional, [H]): the sum over b and t of |eta_t dL/dalpha_t|,
 * the mass of the terms dlambda sums (the scale of its rounding error). */
int oracle_bwd(int variant, int pairing, int phi, const double *q, const double *k, const double *v,
               const double *beta, const double *lambda, double eps, int window, int B, int H, int L, int dk, int dv,
               const double *dout, const double *dstate, double *dq, double *dkk, double *dvv, double *dbeta,
               double *dlambda, int nthreads, double *dlambda_l1)
{
    if (variant < 0 || variant > 5) return -2;
    if (B < 0 || H < 0 || L < 0 || dk <= 0 || dv <= 0) return -3;
    if (is_window(variant) && window < 1) return -6;
    double *dlam_bh = (double *)calloc((size_t)B * H + 1, sizeof(double));
    double *dlam_l1_bh = (double *)calloc((size_t)B * H + 1, sizeof(double));
    bwd_job_t J = {variant, pairing, phi, B, H, L, dk, dv, is_window(variant) ? window : 1, eps,
                   q, k, v, beta, lambda, dout, dstate, dq, dkk, dvv, dbeta, dlam_bh, dlam_l1_bh};
    if (nthreads <= 0) nthreads = (int)sysconf(_SC_NPROCESSORS_ONLN);
    if (nthreads < 1) nthreads = 1;
    const int units = B * H;
    if (nthreads > units) nthreads = units > 0 ? units : 1;
    pthread_t *th = (pthread_t *)malloc(sizeof(pthread_t) * nthreads);
    bwd_worker_t *ws = (bwd_worker_t *)malloc(sizeof(bwd_worker_t) * nthreads);
    for (int i = 0; i < nthreads; ++i) {
        ws[i].J = &J; ws[i].tid = i; ws[i].nthreads = nthreads;
        pthread_create(&th[i], NULL, bwd_worker, &ws[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    for (int hh = 0; hh < H; ++hh) {
        double s = 0.0, a = 0.0;
        for (int bb = 0; bb < B; ++bb) {
            s += dlam_bh[(size_t)bb * H + hh];
            a += dlam_l1_bh[(size_t)bb * H + hh];
        }
        dlambda[hh] = s;
        if (dlambda_l1) dlambda_l1[hh] = a;
    }
    free(th); free(ws); free(dlam_bh); free(dlam_l1_bh);
    return nthreads;
}

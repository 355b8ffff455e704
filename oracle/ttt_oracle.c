/*
 * ttt_oracle.c -- CPU oracle for the Test-Time-Training (TTT) layer forward pass.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing in the product path may link, load or call
 * this file; only the test suite, the smoke check and the benchmark's CPU
 * baseline use it. It shares no code, header, table or helper with the CUDA
 * library and includes nothing from it.
 *
 * Plain, slow and obviously correct: double precision throughout, one token at
 * a time, no blocking or fusion. Sources (the TTT pages):
 *   - "Test-Time Training: Linear Complexity Beyond Attention",
 *     section "The Dual-Loop Structure": the inner loop is online gradient
 *     descent on the fast weight, W_t = W_{t-1} - eta * grad l(W_{t-1}; x_t).
 *   - same page, "Key Architectural Mechanics of TTT-Linear", part 1: the
 *     reconstruction loss l(W; x_t) = 1/2 || f(k_t; W) - v_t ||^2.
 *   - part 2: the closed-form gradient (W k - v) k^T of the linear map and the
 *     update with step size eta.
 *   - part 3: the read-out z_t = f(q_t; W_t) uses the weight AFTER token t's
 *     update; LayerNorm plus a residual connection follow (LN(z) + q).
 *   - part 4 "Mini-Batch Parallelism (Dual Formulation)": tokens are grouped in
 *     mini-batches of b; inside a mini-batch every gradient is taken at the
 *     weight the mini-batch starts from, and the accumulated change is carried
 *     to the next mini-batch.
 *   - the page's PyTorch listing (TTTLinearLayer.step): update first, then
 *     evaluate the query; LayerNorm with its default eps 1e-5 and biased
 *     variance.
 *   - "How to Master Test-Time Training for LLMs" and "...for Infinite Context
 *     LLMs": the fast weight may be a small multi-layer perceptron.
 *   - "Test-Time Training Done Right" (abstract): large-chunk TTT, where a chunk's
 *     outputs use the weight of the previous chunks and the weight is then
 *     updated once from the whole chunk.
 *
 * Conventions (row form): f(k; W) = k W with W[d_in][d_out]; the pages' column
 * form W k is the same map with W transposed. All tensors are row-major:
 * Q, K, V, Z are [B][H][T][d]; eta is [B][H][T]; a fast weight is [H][..] when
 * shared across the batch or [B][H][..] per sequence; gamma, beta are [H][d].
 * Readings where the pages are silent (all stated again in the design notes):
 * the loss carries the 1/2; a mini-batch's gradients are summed, each scaled by
 * the step size of the token it comes from; LayerNorm eps and parameters are
 * fixed per head; GELU is the exact erf form.
 */
#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#ifndef M_PI
#define M_PI 3.14159265358979323846
#endif

/* ------------------------------------------------------------------------ */
/* Small dense helpers (row-major, double).                                  */

/* y[j] = sum_i x[i] * A[i][j];  A is n x m. */
static void vec_mat(const double *x, const double *A, int n, int m, double *y) {
    for (int j = 0; j < m; ++j) y[j] = 0.0;
    for (int i = 0; i < n; ++i) {
        const double xi = x[i];
        const double *row = A + (size_t)i * m;
        for (int j = 0; j < m; ++j) y[j] += xi * row[j];
    }
}

static double dot(const double *a, const double *b, int n) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += a[i] * b[i];
    return s;
}

/* ------------------------------------------------------------------------ */
/* LayerNorm over one row of d values (population variance, eps inside the
 * square root), as torch's nn.LayerNorm computes it.                        */

static double ln_forward(const double *x, const double *gamma, const double *beta, int d,
                         double eps, double *xhat, double *y) {
    double mu = 0.0;
    for (int j = 0; j < d; ++j) mu += x[j];
    mu /= d;
    double var = 0.0;
    for (int j = 0; j < d; ++j) var += (x[j] - mu) * (x[j] - mu);
    var /= d;
    const double sigma = sqrt(var + eps);
    for (int j = 0; j < d; ++j) {
        xhat[j] = (x[j] - mu) / sigma;
        y[j] = gamma[j] * xhat[j] + beta[j];
    }
    return sigma;
}

/* Gradient of a loss through y = gamma * xhat + beta back to x, given the
 * gradient gy wrt y:  gx = (ghat - mean(ghat) - xhat * mean(ghat * xhat)) / sigma
 * with ghat = gamma * gy (chain rule through the mean and the variance). */
static void ln_backward(const double *xhat, double sigma, const double *gamma, const double *gy,
                        int d, double *ghat, double *gx) {
    double m1 = 0.0, m2 = 0.0;
    for (int j = 0; j < d; ++j) {
        ghat[j] = gamma[j] * gy[j];
        m1 += ghat[j];
        m2 += ghat[j] * xhat[j];
    }
    m1 /= d;
    m2 /= d;
    for (int j = 0; j < d; ++j) gx[j] = (ghat[j] - m1 - xhat[j] * m2) / sigma;
}

/* GELU(h) = h * Phi(h) with Phi the standard normal CDF (exact erf form). */
double orc_gelu(double h) { return h * 0.5 * (1.0 + erf(h / sqrt(2.0))); }

/* d GELU / dh = Phi(h) + h * phi(h), phi the standard normal density. */
double orc_gelu_prime(double h) {
    const double Phi = 0.5 * (1.0 + erf(h / sqrt(2.0)));
    const double phi = exp(-0.5 * h * h) / sqrt(2.0 * M_PI);
    return Phi + h * phi;
}

/* ------------------------------------------------------------------------ */
/* Per-token work for the linear fast weight.                                */

typedef struct {
    int d, dh;
    double *x, *xhat, *y, *g, *ghat, *gx, *h, *a, *ga, *gh, *z;
} scratch_t;

static void scratch_init(scratch_t *s, int d, int dh) {
    const int n = (dh > d ? dh : d);
    s->d = d;
    s->dh = dh;
    double **bufs[] = {&s->x, &s->xhat, &s->y, &s->g, &s->ghat, &s->gx,
                       &s->h, &s->a, &s->ga, &s->gh, &s->z};
    for (size_t i = 0; i < sizeof(bufs) / sizeof(bufs[0]); ++i)
        *bufs[i] = (double *)calloc((size_t)n, sizeof(double));
}

static void scratch_free(scratch_t *s) {
    double *bufs[] = {s->x, s->xhat, s->y, s->g, s->ghat, s->gx, s->h, s->a, s->ga, s->gh, s->z};
    for (size_t i = 0; i < sizeof(bufs) / sizeof(bufs[0]); ++i) free(bufs[i]);
}

/* f(k; W) for the linear fast weight: k W, or k + LN(k W) when ln != 0.
 * Leaves x = k W, and (for ln) xhat and sigma, in the scratch. */
static double linear_f(const double *k, const double *W, const double *gamma,
                       const double *beta, int d, int ln, double eps, scratch_t *s,
                       double *f) {
    vec_mat(k, W, d, d, s->x);
    if (!ln) {
        for (int j = 0; j < d; ++j) f[j] = s->x[j];
        return 0.0;
    }
    const double sigma = ln_forward(s->x, gamma, beta, d, eps, s->xhat, s->y);
    for (int j = 0; j < d; ++j) f[j] = k[j] + s->y[j];
    return sigma;
}

/* Reconstruction loss l = 1/2 ||f(k; W) - v||^2 for one token. */
double orc_loss_linear(const double *k, const double *v, const double *W, const double *gamma,
                       const double *beta, int d, int ln, double eps) {
    scratch_t s;
    scratch_init(&s, d, 0);
    double *f = (double *)calloc((size_t)d, sizeof(double));
    linear_f(k, W, gamma, beta, d, ln, eps, &s, f);
    double l = 0.0;
    for (int j = 0; j < d; ++j) l += 0.5 * (f[j] - v[j]) * (f[j] - v[j]);
    free(f);
    scratch_free(&s);
    return l;
}

/* dl/dx for one token at weight W, where x = k W is the pre-activation. */
static void linear_dloss_dx(const double *k, const double *v, const double *W,
                            const double *gamma, const double *beta, int d, int ln, double eps,
                            scratch_t *s, double *gx) {
    const double sigma = linear_f(k, W, gamma, beta, d, ln, eps, s, s->z);
    for (int j = 0; j < d; ++j) s->g[j] = s->z[j] - v[j]; /* dl/df */
    if (!ln) {
        for (int j = 0; j < d; ++j) gx[j] = s->g[j];
        return;
    }
    /* f = k + y: dl/dy = dl/df, then back through the LayerNorm. */
    ln_backward(s->xhat, sigma, gamma, s->g, d, s->ghat, gx);
}

/* Gamma = dl/dW = k^T (dl/dx): an outer product, Gamma[i][j] = k_i * gx_j. */
static void linear_grad_into(const double *k, const double *v, const double *W,
                             const double *gamma, const double *beta, int d, int ln, double eps,
                             scratch_t *s, double *Gam) {
    linear_dloss_dx(k, v, W, gamma, beta, d, ln, eps, s, s->gx);
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < d; ++j) Gam[(size_t)i * d + j] = k[i] * s->gx[j];
}

void orc_grad_linear(const double *k, const double *v, const double *W, const double *gamma,
                     const double *beta, int d, int ln, double eps, double *Gam) {
    scratch_t s;
    scratch_init(&s, d, 0);
    linear_grad_into(k, v, W, gamma, beta, d, ln, eps, &s, Gam);
    scratch_free(&s);
}

/* ------------------------------------------------------------------------ */
/* Per-token work for the MLP fast weight: f(k) = k + LN(GELU(k W1) W2).      */

static double mlp_f(const double *k, const double *W1, const double *W2, const double *gamma,
                    const double *beta, int d, int dh, double eps, scratch_t *s, double *f) {
    vec_mat(k, W1, d, dh, s->h);
    for (int i = 0; i < dh; ++i) s->a[i] = orc_gelu(s->h[i]);
    vec_mat(s->a, W2, dh, d, s->x);
    const double sigma = ln_forward(s->x, gamma, beta, d, eps, s->xhat, s->y);
    for (int j = 0; j < d; ++j) f[j] = k[j] + s->y[j];
    return sigma;
}

double orc_loss_mlp(const double *k, const double *v, const double *W1, const double *W2,
                    const double *gamma, const double *beta, int d, int dh, double eps) {
    scratch_t s;
    scratch_init(&s, d, dh);
    double *f = (double *)calloc((size_t)d, sizeof(double));
    mlp_f(k, W1, W2, gamma, beta, d, dh, eps, &s, f);
    double l = 0.0;
    for (int j = 0; j < d; ++j) l += 0.5 * (f[j] - v[j]) * (f[j] - v[j]);
    free(f);
    scratch_free(&s);
    return l;
}

/* Gamma1 = dl/dW1 [d][dh], Gamma2 = dl/dW2 [dh][d] by the chain rule. */
static void mlp_grad_into(const double *k, const double *v, const double *W1, const double *W2,
                          const double *gamma, const double *beta, int d, int dh, double eps,
                          scratch_t *s, double *G1, double *G2) {
    const double sigma = mlp_f(k, W1, W2, gamma, beta, d, dh, eps, s, s->z);
    for (int j = 0; j < d; ++j) s->g[j] = s->z[j] - v[j];
    ln_backward(s->xhat, sigma, gamma, s->g, d, s->ghat, s->gx);
    /* x = a W2:  dl/dW2 = a^T gx,  dl/da = gx W2^T. */
    for (int i = 0; i < dh; ++i) {
        for (int j = 0; j < d; ++j) G2[(size_t)i * d + j] = s->a[i] * s->gx[j];
        s->ga[i] = dot(W2 + (size_t)i * d, s->gx, d);
        s->gh[i] = s->ga[i] * orc_gelu_prime(s->h[i]); /* a = GELU(h) */
    }
    /* h = k W1:  dl/dW1 = k^T gh. */
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < dh; ++j) G1[(size_t)i * dh + j] = k[i] * s->gh[j];
}

void orc_grad_mlp(const double *k, const double *v, const double *W1, const double *W2,
                  const double *gamma, const double *beta, int d, int dh, double eps,
                  double *G1, double *G2) {
    scratch_t s;
    scratch_init(&s, d, dh);
    mlp_grad_into(k, v, W1, W2, gamma, beta, d, dh, eps, &s, G1, G2);
    scratch_free(&s);
}

/* ------------------------------------------------------------------------ */
/* Problem description shared by the per-sequence drivers.                   */

typedef struct {
    const double *Q, *K, *V, *eta, *W1_0, *W2_0, *gamma, *beta;
    double *Z, *W1_out, *W2_out;
    int B, H, T, d, dh, b, ln, w0_per_seq;
    double eps;
} problem_t;

static size_t w1_elems(const problem_t *p) { return (size_t)p->d * (p->dh ? p->dh : p->d); }
static size_t w2_elems(const problem_t *p) { return (size_t)p->dh * p->d; }

/* Initial fast weight of sequence `seq` (= batch * H + head). */
static const double *w1_init(const problem_t *p, int seq) {
    const int idx = p->w0_per_seq ? seq : (seq % p->H);
    return p->W1_0 + (size_t)idx * w1_elems(p);
}
static const double *w2_init(const problem_t *p, int seq) {
    const int idx = p->w0_per_seq ? seq : (seq % p->H);
    return p->W2_0 + (size_t)idx * w2_elems(p);
}

/* ------------------------------------------------------------------------ */
/* Linear fast weight, update-then-apply with mini-batches of b (primal).
 * For each mini-batch: every token's gradient is taken at the weight W_m the
 * mini-batch starts from; the running weight after token t is
 * W^(t) = W_m - sum_{s<=t} eta_s Gamma_s, formed explicitly; the read-out is
 * z_t = f(q_t; W^(t)); the next mini-batch starts from the last W^(t).       */
static void linear_primal_seq(const problem_t *p, int seq) {
    const int d = p->d, T = p->T, b = p->b, h = seq % p->H;
    const size_t dd = (size_t)d * d;
    const double *gamma = p->gamma ? p->gamma + (size_t)h * d : NULL;
    const double *beta = p->beta ? p->beta + (size_t)h * d : NULL;
    const double *Q = p->Q + (size_t)seq * T * d, *K = p->K + (size_t)seq * T * d,
                 *V = p->V + (size_t)seq * T * d, *eta = p->eta + (size_t)seq * T;
    double *Z = p->Z + (size_t)seq * T * d;
    double *W = malloc(dd * sizeof(double)), *Wm = malloc(dd * sizeof(double)),
           *Gam = malloc(dd * sizeof(double));
    scratch_t s;
    scratch_init(&s, d, 0);
    memcpy(W, w1_init(p, seq), dd * sizeof(double));
    for (int m0 = 0; m0 < T; m0 += b) {
        memcpy(Wm, W, dd * sizeof(double)); /* W_m; W now holds the running W^(t) */
        const int m1 = m0 + b < T ? m0 + b : T; /* a last mini-batch may be partial */
        for (int t = m0; t < m1; ++t) {
            linear_grad_into(K + (size_t)t * d, V + (size_t)t * d, Wm, gamma, beta, d, p->ln,
                             p->eps, &s, Gam);
            for (size_t e = 0; e < dd; ++e) W[e] -= eta[t] * Gam[e];
            linear_f(Q + (size_t)t * d, W, gamma, beta, d, p->ln, p->eps, &s, Z + (size_t)t * d);
        }
    }
    if (p->W1_out) memcpy(p->W1_out + (size_t)seq * dd, W, dd * sizeof(double));
    scratch_free(&s);
    free(W);
    free(Wm);
    free(Gam);
}

/* Linear fast weight, dual form of the same mini-batch rule: with
 * G'_s = eta_s * dl/dx_s at W_m (rows of a b x d matrix),
 *   Zpre = Q W_m - tril(Q K^T) G'   (tril keeps s <= t),
 *   W_{m+1} = W_m - K^T G'.
 * Used only to check that the two forms agree. */
static void linear_dual_seq(const problem_t *p, int seq) {
    const int d = p->d, T = p->T, b = p->b, h = seq % p->H;
    const size_t dd = (size_t)d * d;
    const double *gamma = p->gamma ? p->gamma + (size_t)h * d : NULL;
    const double *beta = p->beta ? p->beta + (size_t)h * d : NULL;
    const double *Q = p->Q + (size_t)seq * T * d, *K = p->K + (size_t)seq * T * d,
                 *V = p->V + (size_t)seq * T * d, *eta = p->eta + (size_t)seq * T;
    double *Z = p->Z + (size_t)seq * T * d;
    double *W = malloc(dd * sizeof(double));
    double *G = malloc((size_t)b * d * sizeof(double));
    double *zp = malloc((size_t)d * sizeof(double));
    scratch_t s;
    scratch_init(&s, d, 0);
    memcpy(W, w1_init(p, seq), dd * sizeof(double));
    for (int m0 = 0; m0 < T; m0 += b) {
        const int nb = T - m0 < b ? T - m0 : b; /* a last mini-batch may be partial */
        for (int r = 0; r < nb; ++r) {
            const int t = m0 + r;
            linear_dloss_dx(K + (size_t)t * d, V + (size_t)t * d, W, gamma, beta, d, p->ln, p->eps,
                            &s, G + (size_t)r * d);
            for (int j = 0; j < d; ++j) G[(size_t)r * d + j] *= eta[t];
        }
        for (int r = 0; r < nb; ++r) {
            const double *q = Q + (size_t)(m0 + r) * d;
            vec_mat(q, W, d, d, zp);
            for (int sr = 0; sr <= r; ++sr) {
                const double a = dot(q, K + (size_t)(m0 + sr) * d, d);
                for (int j = 0; j < d; ++j) zp[j] -= a * G[(size_t)sr * d + j];
            }
            double *z = Z + (size_t)(m0 + r) * d;
            if (p->ln) {
                ln_forward(zp, gamma, beta, d, p->eps, s.xhat, s.y);
                for (int j = 0; j < d; ++j) z[j] = q[j] + s.y[j];
            } else {
                for (int j = 0; j < d; ++j) z[j] = zp[j];
            }
        }
        for (int r = 0; r < nb; ++r) {
            const double *k = K + (size_t)(m0 + r) * d;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < d; ++j) W[(size_t)i * d + j] -= k[i] * G[(size_t)r * d + j];
        }
    }
    if (p->W1_out) memcpy(p->W1_out + (size_t)seq * dd, W, dd * sizeof(double));
    scratch_free(&s);
    free(W);
    free(G);
    free(zp);
}

/* Linear fast weight, apply-then-update over chunks of b (large-chunk TTT):
 * every output of chunk c uses W_c, the weight left by the chunks before it;
 * then W_{c+1} = W_c - sum_{s in c} eta_s Gamma_s(W_c). */
static void chunk_primal_seq(const problem_t *p, int seq) {
    const int d = p->d, T = p->T, b = p->b, h = seq % p->H;
    const size_t dd = (size_t)d * d;
    const double *gamma = p->gamma ? p->gamma + (size_t)h * d : NULL;
    const double *beta = p->beta ? p->beta + (size_t)h * d : NULL;
    const double *Q = p->Q + (size_t)seq * T * d, *K = p->K + (size_t)seq * T * d,
                 *V = p->V + (size_t)seq * T * d, *eta = p->eta + (size_t)seq * T;
    double *Z = p->Z + (size_t)seq * T * d;
    double *W = malloc(dd * sizeof(double)), *Acc = malloc(dd * sizeof(double)),
           *Gam = malloc(dd * sizeof(double));
    scratch_t s;
    scratch_init(&s, d, 0);
    memcpy(W, w1_init(p, seq), dd * sizeof(double));
    for (int c0 = 0; c0 < T; c0 += b) {
        for (int t = c0; t < c0 + b; ++t)
            linear_f(Q + (size_t)t * d, W, gamma, beta, d, p->ln, p->eps, &s, Z + (size_t)t * d);
        memset(Acc, 0, dd * sizeof(double));
        for (int t = c0; t < c0 + b; ++t) {
            linear_grad_into(K + (size_t)t * d, V + (size_t)t * d, W, gamma, beta, d, p->ln,
                             p->eps, &s, Gam);
            for (size_t e = 0; e < dd; ++e) Acc[e] += eta[t] * Gam[e];
        }
        for (size_t e = 0; e < dd; ++e) W[e] -= Acc[e];
    }
    if (p->W1_out) memcpy(p->W1_out + (size_t)seq * dd, W, dd * sizeof(double));
    scratch_free(&s);
    free(W);
    free(Acc);
    free(Gam);
}

/* MLP fast weight, update-then-apply with mini-batches of b (primal). */
static void mlp_primal_seq(const problem_t *p, int seq) {
    const int d = p->d, dh = p->dh, T = p->T, b = p->b, h = seq % p->H;
    const size_t n1 = w1_elems(p), n2 = w2_elems(p);
    const double *gamma = p->gamma + (size_t)h * d, *beta = p->beta + (size_t)h * d;
    const double *Q = p->Q + (size_t)seq * T * d, *K = p->K + (size_t)seq * T * d,
                 *V = p->V + (size_t)seq * T * d, *eta = p->eta + (size_t)seq * T;
    double *Z = p->Z + (size_t)seq * T * d;
    double *W1 = malloc(n1 * sizeof(double)), *W1m = malloc(n1 * sizeof(double)),
           *G1 = malloc(n1 * sizeof(double));
    double *W2 = malloc(n2 * sizeof(double)), *W2m = malloc(n2 * sizeof(double)),
           *G2 = malloc(n2 * sizeof(double));
    scratch_t s;
    scratch_init(&s, d, dh);
    memcpy(W1, w1_init(p, seq), n1 * sizeof(double));
    memcpy(W2, w2_init(p, seq), n2 * sizeof(double));
    for (int m0 = 0; m0 < T; m0 += b) {
        memcpy(W1m, W1, n1 * sizeof(double));
        memcpy(W2m, W2, n2 * sizeof(double));
        for (int t = m0; t < m0 + b; ++t) {
            mlp_grad_into(K + (size_t)t * d, V + (size_t)t * d, W1m, W2m, gamma, beta, d, dh,
                          p->eps, &s, G1, G2);
            for (size_t e = 0; e < n1; ++e) W1[e] -= eta[t] * G1[e];
            for (size_t e = 0; e < n2; ++e) W2[e] -= eta[t] * G2[e];
            mlp_f(Q + (size_t)t * d, W1, W2, gamma, beta, d, dh, p->eps, &s, Z + (size_t)t * d);
        }
    }
    if (p->W1_out) memcpy(p->W1_out + (size_t)seq * n1, W1, n1 * sizeof(double));
    if (p->W2_out) memcpy(p->W2_out + (size_t)seq * n2, W2, n2 * sizeof(double));
    scratch_free(&s);
    free(W1); free(W1m); free(G1);
    free(W2); free(W2m); free(G2);
}

/* MLP fast weight, dual form (two stages, one per layer):
 *   H = K W1, A = GELU(H), X = A W2; Gx'_s = eta_s dl/dx_s; Gh' = (Gx' W2^T) * GELU'(H)
 *   Hq = Q W1 - tril(Q K^T) Gh',  Aq = GELU(Hq),  Xq = Aq W2 - tril(Aq A^T) Gx'
 *   z = q + LN(Xq);  W1 -= K^T Gh',  W2 -= A^T Gx'.
 * Used only to check that the two forms agree. */
static void mlp_dual_seq(const problem_t *p, int seq) {
    const int d = p->d, dh = p->dh, T = p->T, b = p->b, h = seq % p->H;
    const size_t n1 = w1_elems(p), n2 = w2_elems(p);
    const double *gamma = p->gamma + (size_t)h * d, *beta = p->beta + (size_t)h * d;
    const double *Q = p->Q + (size_t)seq * T * d, *K = p->K + (size_t)seq * T * d,
                 *V = p->V + (size_t)seq * T * d, *eta = p->eta + (size_t)seq * T;
    double *Z = p->Z + (size_t)seq * T * d;
    double *W1 = malloc(n1 * sizeof(double)), *W2 = malloc(n2 * sizeof(double));
    double *Hk = malloc((size_t)b * dh * sizeof(double)), *Ak = malloc((size_t)b * dh * sizeof(double));
    double *Gx = malloc((size_t)b * d * sizeof(double)), *Gh = malloc((size_t)b * dh * sizeof(double));
    double *hq = malloc((size_t)dh * sizeof(double)), *aq = malloc((size_t)dh * sizeof(double));
    double *xq = malloc((size_t)d * sizeof(double));
    scratch_t s;
    scratch_init(&s, d, dh);
    memcpy(W1, w1_init(p, seq), n1 * sizeof(double));
    memcpy(W2, w2_init(p, seq), n2 * sizeof(double));
    for (int m0 = 0; m0 < T; m0 += b) {
        for (int r = 0; r < b; ++r) {
            const int t = m0 + r;
            const double *k = K + (size_t)t * d, *v = V + (size_t)t * d;
            const double sigma = mlp_f(k, W1, W2, gamma, beta, d, dh, p->eps, &s, s.z);
            for (int j = 0; j < d; ++j) s.g[j] = s.z[j] - v[j];
            ln_backward(s.xhat, sigma, gamma, s.g, d, s.ghat, Gx + (size_t)r * d);
            for (int j = 0; j < d; ++j) Gx[(size_t)r * d + j] *= eta[t];
            for (int i = 0; i < dh; ++i) {
                Hk[(size_t)r * dh + i] = s.h[i];
                Ak[(size_t)r * dh + i] = s.a[i];
                Gh[(size_t)r * dh + i] =
                    dot(W2 + (size_t)i * d, Gx + (size_t)r * d, d) * orc_gelu_prime(s.h[i]);
            }
        }
        for (int r = 0; r < b; ++r) {
            const double *q = Q + (size_t)(m0 + r) * d;
            vec_mat(q, W1, d, dh, hq);
            for (int sr = 0; sr <= r; ++sr) {
                const double a = dot(q, K + (size_t)(m0 + sr) * d, d);
                for (int i = 0; i < dh; ++i) hq[i] -= a * Gh[(size_t)sr * dh + i];
            }
            for (int i = 0; i < dh; ++i) aq[i] = orc_gelu(hq[i]);
            vec_mat(aq, W2, dh, d, xq);
            for (int sr = 0; sr <= r; ++sr) {
                const double a = dot(aq, Ak + (size_t)sr * dh, dh);
                for (int j = 0; j < d; ++j) xq[j] -= a * Gx[(size_t)sr * d + j];
            }
            ln_forward(xq, gamma, beta, d, p->eps, s.xhat, s.y);
            double *z = Z + (size_t)(m0 + r) * d;
            for (int j = 0; j < d; ++j) z[j] = q[j] + s.y[j];
        }
        for (int r = 0; r < b; ++r) {
            const double *k = K + (size_t)(m0 + r) * d;
            for (int i = 0; i < d; ++i)
                for (int j = 0; j < dh; ++j) W1[(size_t)i * dh + j] -= k[i] * Gh[(size_t)r * dh + j];
            for (int i = 0; i < dh; ++i)
                for (int j = 0; j < d; ++j)
                    W2[(size_t)i * d + j] -= Ak[(size_t)r * dh + i] * Gx[(size_t)r * d + j];
        }
    }
    if (p->W1_out) memcpy(p->W1_out + (size_t)seq * n1, W1, n1 * sizeof(double));
    if (p->W2_out) memcpy(p->W2_out + (size_t)seq * n2, W2, n2 * sizeof(double));
    scratch_free(&s);
    free(W1); free(W2); free(Hk); free(Ak); free(Gx); free(Gh); free(hq); free(aq); free(xq);
}

/* ------------------------------------------------------------------------ */
/* Threaded driver over independent sequences (plain pthreads work queue).  */

typedef void (*seq_fn)(const problem_t *, int);

typedef struct {
    const problem_t *p;
    seq_fn fn;
    const int *seqs;
    int nseqs;
    volatile int next;
} queue_t;

static void *worker(void *arg) {
    queue_t *q = (queue_t *)arg;
    for (;;) {
        const int i = __sync_fetch_and_add(&q->next, 1);
        if (i >= q->nseqs) break;
        q->fn(q->p, q->seqs ? q->seqs[i] : i);
    }
    return NULL;
}

int orc_num_threads(void) {
    long n = sysconf(_SC_NPROCESSORS_ONLN);
    return n > 0 ? (int)n : 1;
}

static void linear_primal_seq(const problem_t *p, int seq);
static void linear_dual_seq(const problem_t *p, int seq);

static int run(const problem_t *p, seq_fn fn, const int *seqs, int nseqs, int nthreads) {
    if (p->b <= 0 || p->d <= 0) return -2;
    /* Only the linear forms define a partial last mini-batch (fewer tokens). */
    if (p->T % p->b != 0 && fn != linear_primal_seq && fn != linear_dual_seq) return -2;
    const int total = p->B * p->H;
    if (!seqs) nseqs = total;
    for (int i = 0; seqs && i < nseqs; ++i)
        if (seqs[i] < 0 || seqs[i] >= total) return -1;
    if (nthreads <= 0) nthreads = orc_num_threads();
    if (nthreads > nseqs) nthreads = nseqs > 0 ? nseqs : 1;
    queue_t q = {p, fn, seqs, nseqs, 0};
    if (nthreads == 1) {
        worker(&q);
        return 0;
    }
    pthread_t *th = malloc((size_t)nthreads * sizeof(pthread_t));
    for (int i = 0; i < nthreads; ++i) pthread_create(&th[i], NULL, worker, &q);
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
    free(th);
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Exported entry points. `seqs` (may be NULL = all) lists the sequences
 * (batch * H + head) to compute; the others are left untouched. Return 0 on
 * success, -1 bad sequence index, -2 bad shape.                             */

#define PROBLEM(...) problem_t p = {__VA_ARGS__}

int orc_linear_primal(const double *Q, const double *K, const double *V, const double *eta,
                      const double *W0, const double *gamma, const double *beta, double *Z,
                      double *W_out, int B, int H, int T, int d, int b, int ln, int w0_per_seq,
                      double eps, const int *seqs, int nseqs, int nthreads) {
    PROBLEM(Q, K, V, eta, W0, NULL, gamma, beta, Z, W_out, NULL, B, H, T, d, 0, b, ln,
            w0_per_seq, eps);
    return run(&p, linear_primal_seq, seqs, nseqs, nthreads);
}

int orc_linear_dual(const double *Q, const double *K, const double *V, const double *eta,
                    const double *W0, const double *gamma, const double *beta, double *Z,
                    double *W_out, int B, int H, int T, int d, int b, int ln, int w0_per_seq,
                    double eps, const int *seqs, int nseqs, int nthreads) {
    PROBLEM(Q, K, V, eta, W0, NULL, gamma, beta, Z, W_out, NULL, B, H, T, d, 0, b, ln,
            w0_per_seq, eps);
    return run(&p, linear_dual_seq, seqs, nseqs, nthreads);
}

int orc_chunk_primal(const double *Q, const double *K, const double *V, const double *eta,
                     const double *W0, const double *gamma, const double *beta, double *Z,
                     double *W_out, int B, int H, int T, int d, int chunk, int ln, int w0_per_seq,
                     double eps, const int *seqs, int nseqs, int nthreads) {
    PROBLEM(Q, K, V, eta, W0, NULL, gamma, beta, Z, W_out, NULL, B, H, T, d, 0, chunk, ln,
            w0_per_seq, eps);
    return run(&p, chunk_primal_seq, seqs, nseqs, nthreads);
}

int orc_mlp_primal(const double *Q, const double *K, const double *V, const double *eta,
                   const double *W1_0, const double *W2_0, const double *gamma,
                   const double *beta, double *Z, double *W1_out, double *W2_out, int B, int H,
                   int T, int d, int dh, int b, int w0_per_seq, double eps, const int *seqs,
                   int nseqs, int nthreads) {
    PROBLEM(Q, K, V, eta, W1_0, W2_0, gamma, beta, Z, W1_out, W2_out, B, H, T, d, dh, b, 1,
            w0_per_seq, eps);
    return run(&p, mlp_primal_seq, seqs, nseqs, nthreads);
}

int orc_mlp_dual(const double *Q, const double *K, const double *V, const double *eta,
                 const double *W1_0, const double *W2_0, const double *gamma, const double *beta,
                 double *Z, double *W1_out, double *W2_out, int B, int H, int T, int d, int dh,
                 int b, int w0_per_seq, double eps, const int *seqs, int nseqs, int nthreads) {
    PROBLEM(Q, K, V, eta, W1_0, W2_0, gamma, beta, Z, W1_out, W2_out, B, H, T, d, dh, b, 1,
            w0_per_seq, eps);
    return run(&p, mlp_dual_seq, seqs, nseqs, nthreads);
}

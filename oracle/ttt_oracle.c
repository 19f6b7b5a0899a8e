/*
 * Float64 CPU oracle for the TTT layer inner-loop forward.
 *
 * TEST INFRASTRUCTURE, NOT PART OF THE PRODUCT.  Only the test suite, the
 * smoke check and the benchmark's CPU-baseline leg may load this library.  It
 * shares no code, header or constant with the CUDA path.
 *
 * What it computes (paper: "Learning to (Learn at Test Time): RNNs with
 * Expressive Hidden States"; the passages are those of the paper digest on
 * equinox-blog, "论文速览 | TTT"):
 *
 *   - Naive TTT, update then output (section 3.1):
 *         W_t = W_{t-1} - eta * grad l(W_{t-1}; x_t),   z_t = f(x_t; W_t)
 *   - Multi-view reconstruction loss and output rule (section 3.3):
 *         l(W; x_t) = || f(theta_K x_t; W) - theta_V x_t ||^2,
 *         z_t = f(theta_Q x_t; W_t)
 *     The inner-loop routines receive q_t, k_t, v_t directly; the views
 *     themselves, with the learning-rate gate below, are computed from the
 *     layer input x by ttt_oracle_qkv_prologue (the fused prologue).
 *   - Learnable inner learning rate (section 4.6):
 *         eta(x) = eta_base * sigmoid(theta_lr^T x),
 *     one theta_lr vector per head.
 *   - Mini-batch gradient descent (section 3.5): inside a mini-batch of b
 *     tokens every gradient is taken at the state W_{t'} of the batch start,
 *     and the updates are applied cumulatively token by token:
 *         G_t = grad l(W_{t'}; x_t),   W_t = W_{t-1} - eta_t G_t.
 *     This is written out literally (the "primal" form); the dual form of
 *     sections 3.6-3.7 is an algebraic rewrite of the same result and is the
 *     GPU's route, not the oracle's.
 *   - Inner models (section 4.4): linear f(x) = x W; LN+residual
 *     f(x) = x + LN(x W + c); two-layer MLP f(x) = GELU(x W1 + c1) W2 + c2
 *     with hidden size 4d, optionally with LN+residual on its output layer,
 *     f(x) = x + LN(GELU(x W1 + c1) W2 + c2).
 *   - Learnable per-token learning rate (section 4.6): eta_t is an input, one
 *     value per token, scaling that token's own gradient.
 *   - Decode / generate uses the primal form one token at a time (section
 *     6.11): the b = 1 update followed by the output.
 *   - Outer-loop gradients (section 3.4: the outer loop trains the
 *     projections, the initial state and the learning-rate parameters with
 *     gradients that pass through the inner loop's updates):
 *     the backward of the TTT-Linear forward, plain and LN+residual (there
 *     also the initial bias and the LN parameters), and of the TTT-MLP
 *     forward, is reverse-mode differentiation of the same primal loop,
 *     token by token.
 *
 * Readings of points the pages leave open (each one is listed in the design
 * notes of the repository):
 *   - Row-vector convention f(x) = x W (W is d_in x d_out).
 *   - Half-loss gradient: grad of 1/2 ||f - v||^2.  The pages' dual form
 *     carries a factor 2 that is folded into eta.
 *   - Biases c, c1, c2 are parameters of f and are part of the state:
 *     updated by the same gradient step and returned.
 *   - LN uses the biased variance over the d features and eps = ln_eps;
 *     gamma and beta are fixed during the inner loop.
 *   - GELU is the exact erf form x * Phi(x).
 *   - A short last mini-batch (T not a multiple of b) follows the same rules.
 *
 * Layouts (all row-major, float64):
 *   Q, K, V, Z : [B, H, T, d]          eta : [B, H, T]
 *   W0         : unit (n, h) reads W0 + n * W0_bstride + h * d * d   (d x d)
 *   c0, gamma, beta : [H, d] (c0 with the same batch-stride rule, may be NULL)
 *   W_out      : [B, H, d, d]          c_out : [B, H, d] (may be NULL)
 *   MLP: W1 [.., d, 4d], c1 [.., 4d], W2 [.., 4d, d], c2 [.., d]
 *
 * Parallel over (sequence, head) units with OpenMP; each unit is computed
 * serially in the order written above.
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static double gelu(double x) { return 0.5 * x * (1.0 + erf(x / sqrt(2.0))); }

/* d/dx [x Phi(x)] = Phi(x) + x phi(x) */
static double gelu_grad(double x) {
    const double Phi = 0.5 * (1.0 + erf(x / sqrt(2.0)));
    const double phi = exp(-0.5 * x * x) / sqrt(2.0 * M_PI);
    return Phi + x * phi;
}

/* y[j] = sum_i x[i] W[i][j]  (x: n_in, W: n_in x n_out) */
static void vec_mat(int n_in, int n_out, const double *x, const double *W, double *y) {
    for (int j = 0; j < n_out; ++j) y[j] = 0.0;
    for (int i = 0; i < n_in; ++i) {
        const double xi = x[i];
        const double *Wi = W + (size_t)i * n_out;
        for (int j = 0; j < n_out; ++j) y[j] += xi * Wi[j];
    }
}

/* LayerNorm over n features, biased variance.  Writes xhat and returns r = 1/sqrt(var+eps). */
static double layer_norm(int n, const double *y, double eps, double *xhat) {
    double mu = 0.0;
    for (int j = 0; j < n; ++j) mu += y[j];
    mu /= n;
    double var = 0.0;
    for (int j = 0; j < n; ++j) var += (y[j] - mu) * (y[j] - mu);
    var /= n;
    const double r = 1.0 / sqrt(var + eps);
    for (int j = 0; j < n; ++j) xhat[j] = (y[j] - mu) * r;
    return r;
}

/* f(x; W, c) for the linear / LN+residual inner model. */
static void linear_model_forward(int d, const double *x, const double *W, const double *c, int use_ln,
                                 const double *gamma, const double *beta, double eps, double *out,
                                 double *tmp_y, double *tmp_xh) {
    vec_mat(d, d, x, W, tmp_y);
    if (!use_ln) {
        for (int j = 0; j < d; ++j) out[j] = tmp_y[j];
        return;
    }
    for (int j = 0; j < d; ++j) tmp_y[j] += c[j];
    layer_norm(d, tmp_y, eps, tmp_xh);
    for (int j = 0; j < d; ++j) out[j] = x[j] + gamma[j] * tmp_xh[j] + beta[j];
}

/*
 * LN+residual output f = x + gamma * LN(y) + beta over d features: the
 * gradient of 1/2 || f - v ||^2 with respect to y (x is the model's input).
 */
static void ln_residual_delta(int d, const double *x, const double *v, const double *y, const double *gamma,
                              const double *beta, double eps, double *delta, double *xh) {
    const double r = layer_norm(d, y, eps, xh);
    /* e = f(k) - v ; g = dL/dxhat = gamma * e */
    double mean_g = 0.0, mean_gx = 0.0;
    for (int j = 0; j < d; ++j) {
        const double e = x[j] + gamma[j] * xh[j] + beta[j] - v[j];
        const double g = gamma[j] * e;
        delta[j] = g; /* keep g for now */
        mean_g += g;
        mean_gx += g * xh[j];
    }
    mean_g /= d;
    mean_gx /= d;
    /* backward through xhat = (y - mu) r */
    for (int j = 0; j < d; ++j) delta[j] = r * (delta[j] - mean_g - xh[j] * mean_gx);
}

/*
 * Gradient of 1/2 || f(k; W, c) - v ||^2 with respect to the pre-activation
 * y = k W (+ c).  grad_W = k^T delta, grad_c = delta.
 */
static void linear_model_delta(int d, const double *k, const double *v, const double *W, const double *c,
                               int use_ln, const double *gamma, const double *beta, double eps,
                               double *delta, double *y, double *xh) {
    vec_mat(d, d, k, W, y);
    if (!use_ln) {
        for (int j = 0; j < d; ++j) delta[j] = y[j] - v[j];
        return;
    }
    for (int j = 0; j < d; ++j) y[j] += c[j];
    ln_residual_delta(d, k, v, y, gamma, beta, eps, delta, xh);
}

static void linear_unit(int T, int d, int b, const double *Q, const double *K, const double *V,
                        const double *eta, const double *W0, const double *c0, int use_ln, const double *gamma,
                        const double *beta, double eps, double *Z, double *W_out, double *c_out) {
    const size_t dd = (size_t)d * d;
    double *Ws = malloc(dd * sizeof(double));   /* state at the mini-batch start */
    double *Wc = malloc(dd * sizeof(double));   /* running state W_t */
    double *cs = calloc(d, sizeof(double));
    double *cc = calloc(d, sizeof(double));
    double *delta = malloc(d * sizeof(double));
    double *y = malloc(d * sizeof(double));
    double *xh = malloc(d * sizeof(double));
    memcpy(Wc, W0, dd * sizeof(double));
    if (c0) memcpy(cc, c0, d * sizeof(double));

    for (int t0 = 0; t0 < T; t0 += b) {
        const int t1 = (t0 + b < T) ? t0 + b : T;
        memcpy(Ws, Wc, dd * sizeof(double));
        memcpy(cs, cc, d * sizeof(double));
        for (int t = t0; t < t1; ++t) {
            const double *k = K + (size_t)t * d, *v = V + (size_t)t * d, *q = Q + (size_t)t * d;
            /* gradient at the batch-start state */
            linear_model_delta(d, k, v, Ws, cs, use_ln, gamma, beta, eps, delta, y, xh);
            /* cumulative update W_t = W_{t-1} - eta_t G_t */
            const double et = eta[t];
            for (int i = 0; i < d; ++i) {
                const double a = et * k[i];
                double *Wi = Wc + (size_t)i * d;
                for (int j = 0; j < d; ++j) Wi[j] -= a * delta[j];
            }
            if (use_ln)
                for (int j = 0; j < d; ++j) cc[j] -= et * delta[j];
            /* output with the updated state */
            linear_model_forward(d, q, Wc, cc, use_ln, gamma, beta, eps, Z + (size_t)t * d, y, xh);
        }
    }
    memcpy(W_out, Wc, dd * sizeof(double));
    if (c_out) memcpy(c_out, cc, d * sizeof(double));
    free(Ws); free(Wc); free(cs); free(cc); free(delta); free(y); free(xh);
}

int ttt_oracle_linear_forward(int B, int H, int T, int d, int b, const double *Q, const double *K,
                              const double *V, const double *eta, const double *W0, long long W0_bstride,
                              const double *c0, long long c0_bstride, int use_ln, const double *gamma,
                              const double *beta, double eps, double *Z, double *W_out, double *c_out,
                              int nthreads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0) return 1;
    if (!W0 || !W_out || (T > 0 && (!Q || !K || !V || !eta || !Z))) return 1;
    if (use_ln && (!gamma || !beta)) return 1;
    const long long units = (long long)B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long long u = 0; u < units; ++u) {
        const int n = (int)(u / H), h = (int)(u % H);
        const size_t tok = (size_t)u * T * d;
        linear_unit(T, d, b, Q + tok, K + tok, V + tok, eta + (size_t)u * T,
                    W0 + (size_t)n * W0_bstride + (size_t)h * d * d,
                    c0 ? c0 + (size_t)n * c0_bstride + (size_t)h * d : NULL, use_ln,
                    use_ln ? gamma + (size_t)h * d : NULL, use_ln ? beta + (size_t)h * d : NULL, eps,
                    Z + tok, W_out + (size_t)u * d * d, c_out ? c_out + (size_t)u * d : NULL);
    }
    (void)nthreads;
    return 0;
}

/* ---------------------------------------------------------------------------
 * Two-layer MLP inner model f(x) = GELU(x W1 + c1) W2 + c2, hidden size m.
 * ------------------------------------------------------------------------- */
static void mlp_unit(int T, int d, int m, int b, const double *Q, const double *K, const double *V,
                     const double *eta, const double *W1_0, const double *c1_0, const double *W2_0,
                     const double *c2_0, int use_ln, const double *gamma, const double *beta, double eps,
                     double *Z, double *W1_out, double *c1_out, double *W2_out, double *c2_out) {
    const size_t n1 = (size_t)d * m, n2 = (size_t)m * d;
    double *W1s = malloc(n1 * sizeof(double)), *W1c = malloc(n1 * sizeof(double));
    double *W2s = malloc(n2 * sizeof(double)), *W2c = malloc(n2 * sizeof(double));
    double *c1s = malloc(m * sizeof(double)), *c1c = malloc(m * sizeof(double));
    double *c2s = malloc(d * sizeof(double)), *c2c = malloc(d * sizeof(double));
    double *a = malloc(m * sizeof(double)), *hh = malloc(m * sizeof(double));
    double *d1 = malloc(m * sizeof(double)), *e = malloc(d * sizeof(double));
    double *y = malloc(d * sizeof(double)), *xh = malloc(d * sizeof(double));
    memcpy(W1c, W1_0, n1 * sizeof(double));
    memcpy(W2c, W2_0, n2 * sizeof(double));
    if (c1_0) memcpy(c1c, c1_0, m * sizeof(double)); else memset(c1c, 0, m * sizeof(double));
    if (c2_0) memcpy(c2c, c2_0, d * sizeof(double)); else memset(c2c, 0, d * sizeof(double));

    for (int t0 = 0; t0 < T; t0 += b) {
        const int t1 = (t0 + b < T) ? t0 + b : T;
        memcpy(W1s, W1c, n1 * sizeof(double));
        memcpy(W2s, W2c, n2 * sizeof(double));
        memcpy(c1s, c1c, m * sizeof(double));
        memcpy(c2s, c2c, d * sizeof(double));
        for (int t = t0; t < t1; ++t) {
            const double *k = K + (size_t)t * d, *v = V + (size_t)t * d, *q = Q + (size_t)t * d;
            /* forward at the batch-start parameters */
            vec_mat(d, m, k, W1s, a);
            for (int p = 0; p < m; ++p) { a[p] += c1s[p]; hh[p] = gelu(a[p]); }
            if (!use_ln) {
                vec_mat(m, d, hh, W2s, e);
                for (int j = 0; j < d; ++j) e[j] += c2s[j] - v[j];
            } else {
                /* f = k + LN(h W2 + c2): e becomes the gradient with respect to y = h W2 + c2 */
                vec_mat(m, d, hh, W2s, y);
                for (int j = 0; j < d; ++j) y[j] += c2s[j];
                ln_residual_delta(d, k, v, y, gamma, beta, eps, e, xh);
            }
            /* backward: d1 = (e W2^T) * GELU'(a) */
            for (int p = 0; p < m; ++p) {
                double s = 0.0;
                const double *W2p = W2s + (size_t)p * d;
                for (int j = 0; j < d; ++j) s += W2p[j] * e[j];
                d1[p] = s * gelu_grad(a[p]);
            }
            /* cumulative update with this token's gradient */
            const double et = eta[t];
            for (int i = 0; i < d; ++i) {
                const double ak = et * k[i];
                double *row = W1c + (size_t)i * m;
                for (int p = 0; p < m; ++p) row[p] -= ak * d1[p];
            }
            for (int p = 0; p < m; ++p) c1c[p] -= et * d1[p];
            for (int p = 0; p < m; ++p) {
                const double ah = et * hh[p];
                double *row = W2c + (size_t)p * d;
                for (int j = 0; j < d; ++j) row[j] -= ah * e[j];
            }
            for (int j = 0; j < d; ++j) c2c[j] -= et * e[j];
            /* output with the updated parameters */
            vec_mat(d, m, q, W1c, a);
            for (int p = 0; p < m; ++p) hh[p] = gelu(a[p] + c1c[p]);
            double *z = Z + (size_t)t * d;
            vec_mat(m, d, hh, W2c, z);
            for (int j = 0; j < d; ++j) z[j] += c2c[j];
            if (use_ln) {
                layer_norm(d, z, eps, xh);
                for (int j = 0; j < d; ++j) z[j] = q[j] + gamma[j] * xh[j] + beta[j];
            }
        }
    }
    memcpy(W1_out, W1c, n1 * sizeof(double));
    memcpy(W2_out, W2c, n2 * sizeof(double));
    if (c1_out) memcpy(c1_out, c1c, m * sizeof(double));
    if (c2_out) memcpy(c2_out, c2c, d * sizeof(double));
    free(W1s); free(W1c); free(W2s); free(W2c); free(c1s); free(c1c); free(c2s); free(c2c);
    free(a); free(hh); free(d1); free(e); free(y); free(xh);
}

/* TTT-MLP, optionally with LN+residual on the output layer,
 *     f(x) = x + gamma LN(GELU(x W1 + c1) W2 + c2) + beta   (use_ln = 1),
 * the form the pages give for TTT-MLP in practice (section 4.4). */
int ttt_oracle_mlp_ln_forward(int B, int H, int T, int d, int m, int b, const double *Q, const double *K,
                              const double *V, const double *eta, const double *W1, const double *c1,
                              const double *W2, const double *c2, long long p_bstride_scale, int use_ln,
                              const double *gamma, const double *beta, double eps, double *Z, double *W1_out,
                              double *c1_out, double *W2_out, double *c2_out, int nthreads) {
    /* p_bstride_scale = 0: parameters are [H, ...] shared over the batch;
       1: parameters are [B, H, ...] (one set per sequence).  gamma, beta: [H, d]. */
    if (B < 0 || H < 0 || T < 0 || d <= 0 || m <= 0 || b <= 0) return 1;
    if (use_ln && (!gamma || !beta || !(eps > 0.0))) return 1;
    if (!W1 || !W2 || !W1_out || !W2_out || (T > 0 && (!Q || !K || !V || !eta || !Z))) return 1;
    const long long units = (long long)B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long long u = 0; u < units; ++u) {
        const long long pu = p_bstride_scale ? u : (u % H);
        const size_t tok = (size_t)u * T * d;
        const long long hd = u % H;
        mlp_unit(T, d, m, b, Q + tok, K + tok, V + tok, eta + (size_t)u * T, W1 + (size_t)pu * d * m,
                 c1 ? c1 + (size_t)pu * m : NULL, W2 + (size_t)pu * m * d, c2 ? c2 + (size_t)pu * d : NULL,
                 use_ln, use_ln ? gamma + (size_t)hd * d : NULL, use_ln ? beta + (size_t)hd * d : NULL, eps,
                 Z + tok, W1_out + (size_t)u * d * m, c1_out ? c1_out + (size_t)u * m : NULL,
                 W2_out + (size_t)u * m * d, c2_out ? c2_out + (size_t)u * d : NULL);
    }
    (void)nthreads;
    return 0;
}

int ttt_oracle_mlp_forward(int B, int H, int T, int d, int m, int b, const double *Q, const double *K,
                           const double *V, const double *eta, const double *W1, const double *c1,
                           const double *W2, const double *c2, long long p_bstride_scale, double *Z,
                           double *W1_out, double *c1_out, double *W2_out, double *c2_out, int nthreads) {
    return ttt_oracle_mlp_ln_forward(B, H, T, d, m, b, Q, K, V, eta, W1, c1, W2, c2, p_bstride_scale, 0, NULL,
                                     NULL, 1e-6, Z, W1_out, c1_out, W2_out, c2_out, nthreads);
}

/* ---------------------------------------------------------------------------
 * Decode: one token per unit, b = 1 primal step, in place on W [B,H,d,d].
 *   W <- W - eta k^T (k W - v),   z = q W  (after the update)
 * ------------------------------------------------------------------------- */
int ttt_oracle_linear_decode_step(int B, int H, int d, double *W, const double *q, const double *k,
                                  const double *v, const double *eta, double *z) {
    if (B < 0 || H < 0 || d <= 0 || !W || !q || !k || !v || !eta || !z) return 1;
    const long long units = (long long)B * H;
    for (long long u = 0; u < units; ++u) {
        double *Wu = W + (size_t)u * d * d;
        const double *qu = q + (size_t)u * d, *ku = k + (size_t)u * d, *vu = v + (size_t)u * d;
        double *e = malloc(d * sizeof(double));
        vec_mat(d, d, ku, Wu, e);
        for (int j = 0; j < d; ++j) e[j] -= vu[j];
        for (int i = 0; i < d; ++i)
            for (int j = 0; j < d; ++j) Wu[(size_t)i * d + j] -= eta[u] * ku[i] * e[j];
        vec_mat(d, d, qu, Wu, z + (size_t)u * d);
        free(e);
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Backward of the TTT-Linear forward (no LN): reverse-mode differentiation of
 * the primal loop above, token by token, for the outer-loop gradients.
 *
 * The loss is any scalar L of the forward's outputs; the caller passes
 * dZ = dL/dZ [B,H,T,d] and dW_out = dL/dW_out [B,H,d,d] (either may be NULL
 * for zero).  Returned: dQ, dK, dV [B,H,T,d], deta [B,H,T] and dW0 [B,H,d,d]
 * (one per sequence, even when W0 is shared: the caller sums over B).
 *
 * Forward of one mini-batch with batch-start state W_s, token by token:
 *     e_t = k_t W_s - v_t,   W_t = W_{t-1} - eta_t k_t^T e_t,   z_t = q_t W_t.
 * Reverse, with D the gradient with respect to the running state (starting
 * at the gradient with respect to the state after the batch), for
 * t = last .. first:
 *     dq_t  = dz_t W_t^T,             D += q_t^T dz_t
 *     deta_t = -<D, k_t^T e_t>,       de_t = -eta_t k_t D
 *     dk_t  = -eta_t e_t D^T + de_t W_s^T,   dv_t = -de_t
 *     dW_s += k_t^T de_t
 * and the gradient with respect to the batch-start state is D + dW_s.
 * The batch-start states come from a forward re-run; the running states W_t
 * of a mini-batch are recomputed from its start.
 * ------------------------------------------------------------------------- */
static void linear_unit_backward(int T, int d, int b, const double *Q, const double *K, const double *V,
                                 const double *eta, const double *W0, const double *dZ, const double *dWout,
                                 double *dQ, double *dK, double *dV, double *deta, double *dW0) {
    const size_t dd = (size_t)d * d;
    const int nb = (T + b - 1) / b;
    double *starts = malloc((size_t)(nb > 0 ? nb : 1) * dd * sizeof(double));  /* state at each batch start */
    double *Wrun = malloc((size_t)(b + 1) * dd * sizeof(double));               /* W_{t0-1} .. W_{t1-1} */
    double *D = malloc(dd * sizeof(double));
    double *dWs = malloc(dd * sizeof(double));
    double *e = malloc((size_t)b * d * sizeof(double));
    double *de = malloc(d * sizeof(double));
    double *Wc = malloc(dd * sizeof(double));
    /* forward re-run: batch-start states */
    memcpy(Wc, W0, dd * sizeof(double));
    for (int i = 0; i < nb; ++i) {
        const int t0 = i * b, t1 = (t0 + b < T) ? t0 + b : T;
        memcpy(starts + (size_t)i * dd, Wc, dd * sizeof(double));
        for (int t = t0; t < t1; ++t) {
            double *et = e + (size_t)(t - t0) * d;
            vec_mat(d, d, K + (size_t)t * d, starts + (size_t)i * dd, et);
            for (int j = 0; j < d; ++j) et[j] -= V[(size_t)t * d + j];
            for (int a = 0; a < d; ++a)
                for (int j = 0; j < d; ++j) Wc[(size_t)a * d + j] -= eta[t] * K[(size_t)t * d + a] * et[j];
        }
    }
    /* reverse sweep */
    if (dWout) memcpy(D, dWout, dd * sizeof(double));
    else memset(D, 0, dd * sizeof(double));
    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * b, t1 = (t0 + b < T) ? t0 + b : T;
        const double *Ws = starts + (size_t)i * dd;
        /* running states of the batch: Wrun[0] = W_s, Wrun[t - t0 + 1] = W_t */
        memcpy(Wrun, Ws, dd * sizeof(double));
        for (int t = t0; t < t1; ++t) {
            double *et = e + (size_t)(t - t0) * d;
            vec_mat(d, d, K + (size_t)t * d, Ws, et);
            for (int j = 0; j < d; ++j) et[j] -= V[(size_t)t * d + j];
            const double *Wp = Wrun + (size_t)(t - t0) * dd;
            double *Wn = Wrun + (size_t)(t - t0 + 1) * dd;
            for (int a = 0; a < d; ++a)
                for (int j = 0; j < d; ++j)
                    Wn[(size_t)a * d + j] = Wp[(size_t)a * d + j] - eta[t] * K[(size_t)t * d + a] * et[j];
        }
        memset(dWs, 0, dd * sizeof(double));
        for (int t = t1 - 1; t >= t0; --t) {
            const double *q = Q + (size_t)t * d, *k = K + (size_t)t * d;
            const double *dz = dZ ? dZ + (size_t)t * d : NULL;
            const double *Wt = Wrun + (size_t)(t - t0 + 1) * dd;
            const double *et = e + (size_t)(t - t0) * d;
            /* z_t = q_t W_t */
            for (int a = 0; a < d; ++a) {
                double acc = 0.0;
                if (dz)
                    for (int j = 0; j < d; ++j) acc += dz[j] * Wt[(size_t)a * d + j];
                dQ[(size_t)t * d + a] = acc;
            }
            if (dz)
                for (int a = 0; a < d; ++a)
                    for (int j = 0; j < d; ++j) D[(size_t)a * d + j] += q[a] * dz[j];
            /* W_t = W_{t-1} - eta_t k_t^T e_t */
            double ge = 0.0;
            for (int a = 0; a < d; ++a)
                for (int j = 0; j < d; ++j) ge += D[(size_t)a * d + j] * k[a] * et[j];
            deta[t] = -ge;
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int a = 0; a < d; ++a) acc += k[a] * D[(size_t)a * d + j];
                de[j] = -eta[t] * acc;
            }
            for (int a = 0; a < d; ++a) {
                double acc1 = 0.0, acc2 = 0.0;
                for (int j = 0; j < d; ++j) {
                    acc1 += et[j] * D[(size_t)a * d + j];
                    acc2 += de[j] * Ws[(size_t)a * d + j];
                }
                dK[(size_t)t * d + a] = -eta[t] * acc1 + acc2;
            }
            for (int j = 0; j < d; ++j) dV[(size_t)t * d + j] = -de[j];
            /* e_t = k_t W_s - v_t */
            for (int a = 0; a < d; ++a)
                for (int j = 0; j < d; ++j) dWs[(size_t)a * d + j] += k[a] * de[j];
        }
        for (size_t x = 0; x < dd; ++x) D[x] += dWs[x];
    }
    memcpy(dW0, D, dd * sizeof(double));
    free(starts); free(Wrun); free(D); free(dWs); free(e); free(de); free(Wc);
}

int ttt_oracle_linear_backward(int B, int H, int T, int d, int b, const double *Q, const double *K,
                               const double *V, const double *eta, const double *W0, long long W0_bstride,
                               const double *dZ, const double *dW_out, double *dQ, double *dK, double *dV,
                               double *deta, double *dW0, int threads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0 || !Q || !K || !V || !eta || !W0 || !dQ || !dK || !dV ||
        !deta || !dW0)
        return 1;
    const long long units = (long long)B * H;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long long u = 0; u < units; ++u) {
        const long long n = u / H, h = u % H;
        const size_t tok = (size_t)u * T * d;
        linear_unit_backward(T, d, b, Q + tok, K + tok, V + tok, eta + (size_t)u * T,
                             W0 + (size_t)n * W0_bstride + (size_t)h * d * d, dZ ? dZ + tok : NULL,
                             dW_out ? dW_out + (size_t)u * d * d : NULL, dQ + tok, dK + tok, dV + tok,
                             deta + (size_t)u * T, dW0 + (size_t)u * d * d);
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Backward of the LN+residual TTT-Linear forward, f(x) = x + gamma LN(x W + c)
 * + beta: reverse-mode differentiation of the primal loop, token by token.
 * Besides the linear model's gradients it returns dc0 (the initial bias) and
 * dgamma, dbeta (the LN parameters, outer-loop parameters fixed inside the
 * inner loop), each per unit; the caller sums over what it shares.
 *
 * Forward of token t with batch-start state (W_s, c_s) and running (W, c):
 *   y = k W_s + c_s,  xh = (y - mean y) r,  r = 1/sqrt(var y + eps)
 *   e = k + gamma xh + beta - v,  g = gamma e
 *   u = g - mean(g) - xh mean(g xh),  delta = r u
 *   W_t = W_{t-1} - eta k^T delta,  c_t = c_{t-1} - eta delta
 *   p = q W_t + c_t,  xo = LN(p) (with r_o),  z = q + gamma xo + beta
 * Each step below is the adjoint of one of these lines, last to first.
 * ------------------------------------------------------------------------- */

/* adjoint of xh = LN(y) (mean and variance over d, r = 1/sqrt(var + eps)):
   dy = r (dxh - mean(dxh) - xh mean(dxh xh)) */
static void ln_adjoint(int d, const double *xh, double r, const double *dxh, double *dy) {
    double m1 = 0.0, m2 = 0.0;
    for (int j = 0; j < d; ++j) { m1 += dxh[j]; m2 += dxh[j] * xh[j]; }
    m1 /= d;
    m2 /= d;
    for (int j = 0; j < d; ++j) dy[j] = r * (dxh[j] - m1 - xh[j] * m2);
}

static void linear_ln_unit_backward(int T, int d, int b, const double *Q, const double *K, const double *V,
                                    const double *eta, const double *W0, const double *c0, const double *gamma,
                                    const double *beta, double eps, const double *dZ, const double *dWout,
                                    const double *dcout, double *dQ, double *dK, double *dV, double *deta,
                                    double *dW0, double *dc0, double *dgamma, double *dbeta) {
    const size_t dd = (size_t)d * d;
    const int nb = (T + b - 1) / b;
    double *Wst = malloc((size_t)(nb > 0 ? nb : 1) * dd * sizeof(double));   /* batch-start W */
    double *cst = malloc((size_t)(nb > 0 ? nb : 1) * d * sizeof(double));    /* batch-start c */
    double *Wrun = malloc((size_t)(b + 1) * dd * sizeof(double));
    double *crun = malloc((size_t)(b + 1) * d * sizeof(double));
    double *DW = malloc(dd * sizeof(double)), *Dc = malloc(d * sizeof(double));
    double *DWs = malloc(dd * sizeof(double)), *Dcs = malloc(d * sizeof(double));
    /* per token of a batch: xh, r, e, g, u, delta */
    double *xh = malloc((size_t)b * d * sizeof(double)), *rr = malloc((size_t)b * sizeof(double));
    double *ee = malloc((size_t)b * d * sizeof(double)), *gg = malloc((size_t)b * d * sizeof(double));
    double *uu = malloc((size_t)b * d * sizeof(double)), *dl = malloc((size_t)b * d * sizeof(double));
    double *mgx = malloc((size_t)b * sizeof(double));
    double *y = malloc(d * sizeof(double)), *p = malloc(d * sizeof(double)), *xo = malloc(d * sizeof(double));
    double *t1 = malloc(d * sizeof(double)), *t2 = malloc(d * sizeof(double)), *t3 = malloc(d * sizeof(double));
    double *dxh = malloc(d * sizeof(double)), *dy = malloc(d * sizeof(double));
    double *Wc = malloc(dd * sizeof(double)), *cc = malloc(d * sizeof(double));

    /* token forward at the batch start: fills xh, r, e, g, u, delta of row i */
    #define TOKEN_FWD(t, i, Ws, cs)                                                                    \
        do {                                                                                           \
            const double *k_ = K + (size_t)(t) * d, *v_ = V + (size_t)(t) * d;                         \
            vec_mat(d, d, k_, (Ws), y);                                                                \
            for (int j = 0; j < d; ++j) y[j] += (cs)[j];                                               \
            rr[i] = layer_norm(d, y, eps, xh + (size_t)(i) * d);                                       \
            double mg = 0.0, mgx_ = 0.0;                                                               \
            for (int j = 0; j < d; ++j) {                                                              \
                const double x_ = xh[(size_t)(i) * d + j];                                             \
                ee[(size_t)(i) * d + j] = k_[j] + gamma[j] * x_ + beta[j] - v_[j];                     \
                gg[(size_t)(i) * d + j] = gamma[j] * ee[(size_t)(i) * d + j];                          \
                mg += gg[(size_t)(i) * d + j];                                                         \
                mgx_ += gg[(size_t)(i) * d + j] * x_;                                                  \
            }                                                                                          \
            mg /= d;                                                                                   \
            mgx_ /= d;                                                                                 \
            mgx[i] = mgx_;                                                                             \
            for (int j = 0; j < d; ++j) {                                                              \
                const double x_ = xh[(size_t)(i) * d + j];                                             \
                uu[(size_t)(i) * d + j] = gg[(size_t)(i) * d + j] - mg - x_ * mgx_;                    \
                dl[(size_t)(i) * d + j] = rr[i] * uu[(size_t)(i) * d + j];                             \
            }                                                                                          \
        } while (0)

    /* forward re-run: batch-start states */
    memcpy(Wc, W0, dd * sizeof(double));
    if (c0) memcpy(cc, c0, d * sizeof(double)); else memset(cc, 0, d * sizeof(double));
    for (int i = 0; i < nb; ++i) {
        const int t0 = i * b, t1_ = (t0 + b < T) ? t0 + b : T;
        memcpy(Wst + (size_t)i * dd, Wc, dd * sizeof(double));
        memcpy(cst + (size_t)i * d, cc, d * sizeof(double));
        for (int t = t0; t < t1_; ++t) {
            TOKEN_FWD(t, t - t0, Wst + (size_t)i * dd, cst + (size_t)i * d);
            const double *k = K + (size_t)t * d;
            for (int a = 0; a < d; ++a)
                for (int j = 0; j < d; ++j) Wc[(size_t)a * d + j] -= eta[t] * k[a] * dl[(size_t)(t - t0) * d + j];
            for (int j = 0; j < d; ++j) cc[j] -= eta[t] * dl[(size_t)(t - t0) * d + j];
        }
    }
    /* reverse sweep */
    if (dWout) memcpy(DW, dWout, dd * sizeof(double)); else memset(DW, 0, dd * sizeof(double));
    if (dcout) memcpy(Dc, dcout, d * sizeof(double)); else memset(Dc, 0, d * sizeof(double));
    memset(dgamma, 0, d * sizeof(double));
    memset(dbeta, 0, d * sizeof(double));
    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * b, t1_ = (t0 + b < T) ? t0 + b : T;
        const double *Ws = Wst + (size_t)i * dd, *cs = cst + (size_t)i * d;
        /* recompute the batch: per-token quantities and running states */
        memcpy(Wrun, Ws, dd * sizeof(double));
        memcpy(crun, cs, d * sizeof(double));
        for (int t = t0; t < t1_; ++t) {
            const int li = t - t0;
            TOKEN_FWD(t, li, Ws, cs);
            const double *k = K + (size_t)t * d;
            const double *Wp = Wrun + (size_t)li * dd, *cp = crun + (size_t)li * d;
            double *Wn = Wrun + (size_t)(li + 1) * dd, *cn = crun + (size_t)(li + 1) * d;
            for (int a = 0; a < d; ++a)
                for (int j = 0; j < d; ++j)
                    Wn[(size_t)a * d + j] = Wp[(size_t)a * d + j] - eta[t] * k[a] * dl[(size_t)li * d + j];
            for (int j = 0; j < d; ++j) cn[j] = cp[j] - eta[t] * dl[(size_t)li * d + j];
        }
        memset(DWs, 0, dd * sizeof(double));
        memset(Dcs, 0, d * sizeof(double));
        for (int t = t1_ - 1; t >= t0; --t) {
            const int li = t - t0;
            const double *q = Q + (size_t)t * d, *k = K + (size_t)t * d;
            const double *Wt = Wrun + (size_t)(li + 1) * dd, *ct = crun + (size_t)(li + 1) * d;
            const double *xt = xh + (size_t)li * d, *et = ee + (size_t)li * d, *gt = gg + (size_t)li * d;
            const double *ut = uu + (size_t)li * d, *dt = dl + (size_t)li * d;
            double *dq = dQ + (size_t)t * d, *dk = dK + (size_t)t * d, *dv = dV + (size_t)t * d;
            for (int j = 0; j < d; ++j) { dq[j] = 0.0; dk[j] = 0.0; }
            /* z = q + gamma xo + beta, xo = LN(p), p = q W_t + c_t */
            if (dZ) {
                const double *dz = dZ + (size_t)t * d;
                vec_mat(d, d, q, Wt, p);
                for (int j = 0; j < d; ++j) p[j] += ct[j];
                const double ro = layer_norm(d, p, eps, xo);
                for (int j = 0; j < d; ++j) {
                    dq[j] += dz[j];
                    dgamma[j] += dz[j] * xo[j];
                    dbeta[j] += dz[j];
                    t1[j] = gamma[j] * dz[j];
                }
                ln_adjoint(d, xo, ro, t1, t2);   /* t2 = dp */
                for (int a = 0; a < d; ++a) {
                    double acc = 0.0;
                    for (int j = 0; j < d; ++j) acc += t2[j] * Wt[(size_t)a * d + j];
                    dq[a] += acc;
                }
                for (int a = 0; a < d; ++a)
                    for (int j = 0; j < d; ++j) DW[(size_t)a * d + j] += q[a] * t2[j];
                for (int j = 0; j < d; ++j) Dc[j] += t2[j];
            }
            /* W_t = W_{t-1} - eta k^T delta,  c_t = c_{t-1} - eta delta */
            double ge = 0.0;
            for (int j = 0; j < d; ++j) {
                double acc = Dc[j];
                for (int a = 0; a < d; ++a) acc += k[a] * DW[(size_t)a * d + j];
                t3[j] = -eta[t] * acc;   /* t3 = ddelta */
                ge += acc * dt[j];
            }
            deta[t] = -ge;
            for (int a = 0; a < d; ++a) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += dt[j] * DW[(size_t)a * d + j];
                dk[a] += -eta[t] * acc;
            }
            /* delta = r u, u = g - mean(g) - xh mean(g xh) */
            double dr = 0.0;
            for (int j = 0; j < d; ++j) { dr += t3[j] * ut[j]; t1[j] = rr[li] * t3[j]; }   /* t1 = du */
            double mdu = 0.0, mdux = 0.0;
            for (int j = 0; j < d; ++j) { mdu += t1[j]; mdux += t1[j] * xt[j]; }
            mdu /= d;
            mdux /= d;
            for (int j = 0; j < d; ++j) {
                const double dg = t1[j] - mdu - xt[j] * mdux;
                dxh[j] = -t1[j] * mgx[li] - gt[j] * mdux;   /* through the xh of u */
                /* g = gamma e, e = k + gamma xh + beta - v */
                const double de = gamma[j] * dg;
                dgamma[j] += et[j] * dg + xt[j] * de;
                dbeta[j] += de;
                dk[j] += de;
                dv[j] = -de;
                dxh[j] += gamma[j] * de;
            }
            /* xh = LN(y), and r = 1/sqrt(var + eps) in delta = r u: dr/dy_j = -r^2 xh_j / d */
            ln_adjoint(d, xt, rr[li], dxh, dy);
            for (int j = 0; j < d; ++j) dy[j] += dr * (-rr[li] * rr[li] * xt[j] / d);
            /* y = k W_s + c_s */
            for (int a = 0; a < d; ++a) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += dy[j] * Ws[(size_t)a * d + j];
                dk[a] += acc;
            }
            for (int a = 0; a < d; ++a)
                for (int j = 0; j < d; ++j) DWs[(size_t)a * d + j] += k[a] * dy[j];
            for (int j = 0; j < d; ++j) Dcs[j] += dy[j];
        }
        for (size_t x = 0; x < dd; ++x) DW[x] += DWs[x];
        for (int j = 0; j < d; ++j) Dc[j] += Dcs[j];
    }
    #undef TOKEN_FWD
    memcpy(dW0, DW, dd * sizeof(double));
    memcpy(dc0, Dc, d * sizeof(double));
    free(Wst); free(cst); free(Wrun); free(crun); free(DW); free(Dc); free(DWs); free(Dcs);
    free(xh); free(rr); free(ee); free(gg); free(uu); free(dl); free(mgx);
    free(y); free(p); free(xo); free(t1); free(t2); free(t3); free(dxh); free(dy); free(Wc); free(cc);
}

int ttt_oracle_linear_ln_backward(int B, int H, int T, int d, int b, const double *Q, const double *K,
                                  const double *V, const double *eta, const double *W0, long long W0_bstride,
                                  const double *c0, long long c0_bstride, const double *gamma, const double *beta,
                                  double eps, const double *dZ, const double *dW_out, const double *dc_out,
                                  double *dQ, double *dK, double *dV, double *deta, double *dW0, double *dc0,
                                  double *dgamma, double *dbeta, int threads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || b <= 0 || !Q || !K || !V || !eta || !W0 || !gamma || !beta ||
        !(eps > 0.0) || !dQ || !dK || !dV || !deta || !dW0 || !dc0 || !dgamma || !dbeta)
        return 1;
    const long long units = (long long)B * H;
#ifdef _OPENMP
    if (threads > 0) omp_set_num_threads(threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long long u = 0; u < units; ++u) {
        const long long n = u / H, h = u % H;
        const size_t tok = (size_t)u * T * d;
        linear_ln_unit_backward(T, d, b, Q + tok, K + tok, V + tok, eta + (size_t)u * T,
                                W0 + (size_t)n * W0_bstride + (size_t)h * d * d,
                                c0 ? c0 + (size_t)n * c0_bstride + (size_t)h * d : NULL, gamma + (size_t)h * d,
                                beta + (size_t)h * d, eps, dZ ? dZ + tok : NULL,
                                dW_out ? dW_out + (size_t)u * d * d : NULL, dc_out ? dc_out + (size_t)u * d : NULL,
                                dQ + tok, dK + tok, dV + tok, deta + (size_t)u * T, dW0 + (size_t)u * d * d,
                                dc0 + (size_t)u * d, dgamma + (size_t)u * d, dbeta + (size_t)u * d);
    }
    return 0;
}

/* ---------------------------------------------------------------------------
 * Backward of the TTT-MLP forward (no LN): reverse-mode differentiation of
 * the primal loop, token by token.  Returns dQ, dK, dV, deta and the
 * gradients of the initial parameters dW1, dc1, dW2, dc2 (per unit).
 *
 * Forward of token t with batch-start (W1s, c1s, W2s, c2s) and running state:
 *   a = k W1s + c1s,  h = GELU(a),  e = h W2s + c2s - v
 *   m = e W2s^T,  d1 = m * GELU'(a)
 *   W1 -= eta k^T d1,  c1 -= eta d1,  W2 -= eta h^T e,  c2 -= eta e
 *   aq = q W1_t + c1_t,  hq = GELU(aq),  z = hq W2_t + c2_t
 * GELU''(x) = phi(x) (2 - x^2), the derivative of Phi(x) + x phi(x).
 * ------------------------------------------------------------------------- */
static double gelu_grad2(double x) { return exp(-0.5 * x * x) / sqrt(2.0 * M_PI) * (2.0 - x * x); }

static void mlp_unit_backward(int T, int d, int m, int b, const double *Q, const double *K, const double *V,
                              const double *eta, const double *W1_0, const double *c1_0, const double *W2_0,
                              const double *c2_0, const double *dZ, const double *dW1o, const double *dc1o,
                              const double *dW2o, const double *dc2o, double *dQ, double *dK, double *dV,
                              double *deta, double *dW1, double *dc1, double *dW2, double *dc2) {
    const size_t n1 = (size_t)d * m;
    const int nb = (T + b - 1) / b;
    const size_t sz = n1 + m + n1 + d;   /* one state: W1, c1, W2, c2 */
    double *starts = malloc((size_t)(nb > 0 ? nb : 1) * sz * sizeof(double));
    double *run = malloc((size_t)(b + 1) * sz * sizeof(double));   /* running states of a batch */
    double *cur = malloc(sz * sizeof(double));
    double *D = malloc(sz * sizeof(double)), *Ds = malloc(sz * sizeof(double));   /* adjoints */
    double *A = malloc((size_t)b * m * sizeof(double)), *Hh = malloc((size_t)b * m * sizeof(double));
    double *E = malloc((size_t)b * d * sizeof(double)), *Mm = malloc((size_t)b * m * sizeof(double));
    double *D1 = malloc((size_t)b * m * sizeof(double));
    double *aq = malloc(m * sizeof(double)), *hq = malloc(m * sizeof(double)), *dhq = malloc(m * sizeof(double));
    double *dd1 = malloc(m * sizeof(double)), *dmv = malloc(m * sizeof(double)), *dh = malloc(m * sizeof(double));
    double *da = malloc(m * sizeof(double)), *de = malloc(d * sizeof(double));
    #define W1P(x) (x)
    #define C1P(x) ((x) + n1)
    #define W2P(x) ((x) + n1 + m)
    #define C2P(x) ((x) + n1 + m + n1)

    /* batch quantities at the batch-start state S, row i = token t */
    #define BATCH_FWD(t, i, S)                                                                         \
        do {                                                                                           \
            const double *k_ = K + (size_t)(t) * d, *v_ = V + (size_t)(t) * d;                         \
            double *a_ = A + (size_t)(i) * m, *h_ = Hh + (size_t)(i) * m, *e_ = E + (size_t)(i) * d;   \
            vec_mat(d, m, k_, W1P(S), a_);                                                             \
            for (int p = 0; p < m; ++p) { a_[p] += C1P(S)[p]; h_[p] = gelu(a_[p]); }                   \
            vec_mat(m, d, h_, W2P(S), e_);                                                             \
            for (int j = 0; j < d; ++j) e_[j] += C2P(S)[j] - v_[j];                                    \
            for (int p = 0; p < m; ++p) {                                                              \
                double acc = 0.0;                                                                      \
                for (int j = 0; j < d; ++j) acc += W2P(S)[(size_t)p * d + j] * e_[j];                  \
                Mm[(size_t)(i) * m + p] = acc;                                                         \
                D1[(size_t)(i) * m + p] = acc * gelu_grad(a_[p]);                                      \
            }                                                                                          \
        } while (0)
    /* one token's update applied to state X (in place) */
    #define TOKEN_UPD(t, i, X)                                                                         \
        do {                                                                                           \
            const double *k_ = K + (size_t)(t) * d, et_ = eta[t];                                      \
            const double *d1_ = D1 + (size_t)(i) * m, *h_ = Hh + (size_t)(i) * m, *e_ = E + (size_t)(i) * d; \
            for (int a2 = 0; a2 < d; ++a2)                                                             \
                for (int p = 0; p < m; ++p) W1P(X)[(size_t)a2 * m + p] -= et_ * k_[a2] * d1_[p];       \
            for (int p = 0; p < m; ++p) C1P(X)[p] -= et_ * d1_[p];                                     \
            for (int p = 0; p < m; ++p)                                                                \
                for (int j = 0; j < d; ++j) W2P(X)[(size_t)p * d + j] -= et_ * h_[p] * e_[j];          \
            for (int j = 0; j < d; ++j) C2P(X)[j] -= et_ * e_[j];                                      \
        } while (0)

    memcpy(W1P(cur), W1_0, n1 * sizeof(double));
    if (c1_0) memcpy(C1P(cur), c1_0, m * sizeof(double)); else memset(C1P(cur), 0, m * sizeof(double));
    memcpy(W2P(cur), W2_0, n1 * sizeof(double));
    if (c2_0) memcpy(C2P(cur), c2_0, d * sizeof(double)); else memset(C2P(cur), 0, d * sizeof(double));
    for (int i = 0; i < nb; ++i) {
        const int t0 = i * b, t1_ = (t0 + b < T) ? t0 + b : T;
        memcpy(starts + (size_t)i * sz, cur, sz * sizeof(double));
        for (int t = t0; t < t1_; ++t) BATCH_FWD(t, t - t0, starts + (size_t)i * sz);
        for (int t = t0; t < t1_; ++t) TOKEN_UPD(t, t - t0, cur);
    }
    /* adjoint of the final state */
    memset(D, 0, sz * sizeof(double));
    if (dW1o) memcpy(W1P(D), dW1o, n1 * sizeof(double));
    if (dc1o) memcpy(C1P(D), dc1o, m * sizeof(double));
    if (dW2o) memcpy(W2P(D), dW2o, n1 * sizeof(double));
    if (dc2o) memcpy(C2P(D), dc2o, d * sizeof(double));
    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * b, t1_ = (t0 + b < T) ? t0 + b : T;
        const double *S = starts + (size_t)i * sz;
        for (int t = t0; t < t1_; ++t) BATCH_FWD(t, t - t0, S);
        memcpy(run, S, sz * sizeof(double));
        for (int t = t0; t < t1_; ++t) {
            memcpy(run + (size_t)(t - t0 + 1) * sz, run + (size_t)(t - t0) * sz, sz * sizeof(double));
            TOKEN_UPD(t, t - t0, run + (size_t)(t - t0 + 1) * sz);
        }
        memset(Ds, 0, sz * sizeof(double));
        for (int t = t1_ - 1; t >= t0; --t) {
            const int li = t - t0;
            const double *q = Q + (size_t)t * d, *k = K + (size_t)t * d;
            const double *Rt = run + (size_t)(li + 1) * sz;   /* state after token t */
            const double *a = A + (size_t)li * m, *h = Hh + (size_t)li * m, *e = E + (size_t)li * d;
            const double *mm = Mm + (size_t)li * m, *d1 = D1 + (size_t)li * m;
            double *dq = dQ + (size_t)t * d, *dk = dK + (size_t)t * d, *dv = dV + (size_t)t * d;
            for (int j = 0; j < d; ++j) { dq[j] = 0.0; dk[j] = 0.0; }
            /* z = GELU(q W1_t + c1_t) W2_t + c2_t */
            if (dZ) {
                const double *dz = dZ + (size_t)t * d;
                vec_mat(d, m, q, W1P(Rt), aq);
                for (int p = 0; p < m; ++p) { aq[p] += C1P(Rt)[p]; hq[p] = gelu(aq[p]); }
                for (int p = 0; p < m; ++p) {
                    double acc = 0.0;
                    for (int j = 0; j < d; ++j) acc += dz[j] * W2P(Rt)[(size_t)p * d + j];
                    dhq[p] = acc * gelu_grad(aq[p]);   /* d(aq) */
                }
                for (int p = 0; p < m; ++p)
                    for (int j = 0; j < d; ++j) W2P(D)[(size_t)p * d + j] += hq[p] * dz[j];
                for (int j = 0; j < d; ++j) C2P(D)[j] += dz[j];
                for (int a2 = 0; a2 < d; ++a2) {
                    double acc = 0.0;
                    for (int p = 0; p < m; ++p) acc += dhq[p] * W1P(Rt)[(size_t)a2 * m + p];
                    dq[a2] += acc;
                }
                for (int a2 = 0; a2 < d; ++a2)
                    for (int p = 0; p < m; ++p) W1P(D)[(size_t)a2 * m + p] += q[a2] * dhq[p];
                for (int p = 0; p < m; ++p) C1P(D)[p] += dhq[p];
            }
            /* the token's update: W1 -= eta k^T d1, c1 -= eta d1, W2 -= eta h^T e, c2 -= eta e */
            double g = 0.0;
            for (int p = 0; p < m; ++p) {
                double acc = C1P(D)[p];
                for (int a2 = 0; a2 < d; ++a2) acc += k[a2] * W1P(D)[(size_t)a2 * m + p];
                dd1[p] = -eta[t] * acc;
                g += acc * d1[p];
            }
            for (int j = 0; j < d; ++j) {
                double acc = C2P(D)[j];
                for (int p = 0; p < m; ++p) acc += h[p] * W2P(D)[(size_t)p * d + j];
                de[j] = -eta[t] * acc;
                g += acc * e[j];
            }
            deta[t] = -g;
            for (int a2 = 0; a2 < d; ++a2) {
                double acc = 0.0;
                for (int p = 0; p < m; ++p) acc += d1[p] * W1P(D)[(size_t)a2 * m + p];
                dk[a2] += -eta[t] * acc;
            }
            for (int p = 0; p < m; ++p) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += e[j] * W2P(D)[(size_t)p * d + j];
                dh[p] = -eta[t] * acc;
            }
            /* d1 = m * GELU'(a), m = e W2s^T */
            for (int p = 0; p < m; ++p) {
                dmv[p] = dd1[p] * gelu_grad(a[p]);
                da[p] = dd1[p] * mm[p] * gelu_grad2(a[p]);
            }
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int p = 0; p < m; ++p) acc += dmv[p] * W2P(S)[(size_t)p * d + j];
                de[j] += acc;
            }
            for (int p = 0; p < m; ++p)
                for (int j = 0; j < d; ++j) W2P(Ds)[(size_t)p * d + j] += dmv[p] * e[j];
            /* e = h W2s + c2s - v */
            for (int p = 0; p < m; ++p) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += de[j] * W2P(S)[(size_t)p * d + j];
                dh[p] += acc;
            }
            for (int p = 0; p < m; ++p)
                for (int j = 0; j < d; ++j) W2P(Ds)[(size_t)p * d + j] += h[p] * de[j];
            for (int j = 0; j < d; ++j) { C2P(Ds)[j] += de[j]; dv[j] = -de[j]; }
            /* h = GELU(a), a = k W1s + c1s */
            for (int p = 0; p < m; ++p) da[p] += dh[p] * gelu_grad(a[p]);
            for (int a2 = 0; a2 < d; ++a2) {
                double acc = 0.0;
                for (int p = 0; p < m; ++p) acc += da[p] * W1P(S)[(size_t)a2 * m + p];
                dk[a2] += acc;
            }
            for (int a2 = 0; a2 < d; ++a2)
                for (int p = 0; p < m; ++p) W1P(Ds)[(size_t)a2 * m + p] += k[a2] * da[p];
            for (int p = 0; p < m; ++p) C1P(Ds)[p] += da[p];
        }
        for (size_t x = 0; x < sz; ++x) D[x] += Ds[x];
    }
    #undef BATCH_FWD
    #undef TOKEN_UPD
    memcpy(dW1, W1P(D), n1 * sizeof(double));
    memcpy(dc1, C1P(D), m * sizeof(double));
    memcpy(dW2, W2P(D), n1 * sizeof(double));
    memcpy(dc2, C2P(D), d * sizeof(double));
    #undef W1P
    #undef C1P
    #undef W2P
    #undef C2P
    free(starts); free(run); free(cur); free(D); free(Ds); free(A); free(Hh); free(E); free(Mm); free(D1);
    free(aq); free(hq); free(dhq); free(dd1); free(dmv); free(dh); free(da); free(de);
}

int ttt_oracle_mlp_backward(int B, int H, int T, int d, int m, int b, const double *Q, const double *K,
                            const double *V, const double *eta, const double *W1, const double *c1,
                            const double *W2, const double *c2, long long p_bstride_scale, const double *dZ,
                            const double *dW1o, const double *dc1o, const double *dW2o, const double *dc2o,
                            double *dQ, double *dK, double *dV, double *deta, double *dW1, double *dc1,
                            double *dW2, double *dc2, int nthreads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || m <= 0 || b <= 0 || !Q || !K || !V || !eta || !W1 || !W2 ||
        !dQ || !dK || !dV || !deta || !dW1 || !dc1 || !dW2 || !dc2)
        return 1;
    const long long units = (long long)B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long long u = 0; u < units; ++u) {
        const long long pu = p_bstride_scale ? u : (u % H);
        const size_t tok = (size_t)u * T * d;
        mlp_unit_backward(T, d, m, b, Q + tok, K + tok, V + tok, eta + (size_t)u * T, W1 + (size_t)pu * d * m,
                          c1 ? c1 + (size_t)pu * m : NULL, W2 + (size_t)pu * m * d, c2 ? c2 + (size_t)pu * d : NULL,
                          dZ ? dZ + tok : NULL, dW1o ? dW1o + (size_t)u * d * m : NULL,
                          dc1o ? dc1o + (size_t)u * m : NULL, dW2o ? dW2o + (size_t)u * m * d : NULL,
                          dc2o ? dc2o + (size_t)u * d : NULL, dQ + tok, dK + tok, dV + tok, deta + (size_t)u * T,
                          dW1 + (size_t)u * d * m, dc1 + (size_t)u * m, dW2 + (size_t)u * m * d, dc2 + (size_t)u * d);
    }
    (void)nthreads;
    return 0;
}

/*
 * Prologue: the three views and the learning-rate gate of every token and
 * head, from the layer input (sections 3.3 and 4.6).
 *
 *   x        : [B, T, Dm]    the layer input, one row per token
 *   theta_q, theta_k, theta_v : [H * d, Dm]   the pages' column form: the
 *              view of token t is theta x_t, and head h owns the rows
 *              h d .. h d + d - 1
 *   theta_lr : [H, Dm]       one gate vector per head
 *   Q, K, V  : [B, H, T, d]  Q[n, h, t, j] = sum_k theta_q[h d + j, k] x[n, t, k]
 *   eta      : [B, H, T]     eta[n, h, t] = eta_base * sigmoid(theta_lr[h] . x[n, t])
 *
 * eta_base is taken as given: the caller states it in the half-loss
 * convention of the inner-loop routines (twice the pages' value).
 */
static double sigmoid(double u) { return 1.0 / (1.0 + exp(-u)); }

/* one view of one token: out[h T d + j] = sum_k theta[(h d + j) Dm + k] x[k] */
static void project_view(int H, int d, int Dm, const double *theta, const double *x, double *out,
                         size_t head_stride) {
    for (int h = 0; h < H; ++h)
        for (int j = 0; j < d; ++j) {
            const double *row = theta + (size_t)(h * d + j) * Dm;
            double acc = 0.0;
            for (int k = 0; k < Dm; ++k) acc += row[k] * x[k];
            out[(size_t)h * head_stride + j] = acc;
        }
}

int ttt_oracle_qkv_prologue(int B, int T, int Dm, int H, int d, const double *x, const double *theta_q,
                            const double *theta_k, const double *theta_v, const double *theta_lr,
                            double eta_base, double *Q, double *K, double *V, double *eta, int nthreads) {
    if (B < 0 || T < 0 || Dm <= 0 || H < 0 || d <= 0 || !x || !theta_q || !theta_k || !theta_v || !theta_lr ||
        !Q || !K || !V || !eta)
        return 1;
    const long long rows = (long long)B * T;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(static)
#endif
    for (long long r = 0; r < rows; ++r) {
        const long long n = r / T, t = r % T;
        const double *xt = x + (size_t)r * Dm;
        const size_t o = ((size_t)n * H * T + (size_t)t) * d;   /* (n, h = 0, t, 0) */
        const size_t hs = (size_t)T * d;                         /* one head further */
        project_view(H, d, Dm, theta_q, xt, Q + o, hs);
        project_view(H, d, Dm, theta_k, xt, K + o, hs);
        project_view(H, d, Dm, theta_v, xt, V + o, hs);
        for (int h = 0; h < H; ++h) {
            const double *g = theta_lr + (size_t)h * Dm;
            double u = 0.0;
            for (int k = 0; k < Dm; ++k) u += g[k] * xt[k];
            eta[((size_t)n * H + h) * T + t] = eta_base * sigmoid(u);
        }
    }
    (void)nthreads;
    return 0;
}

/*
 * Outer-loop gradients of TTT-MLP with LN+residual on the output layer,
 * f(x) = x + gamma LN(GELU(x W1 + c1) W2 + c2) + beta (section 4.4; section 3.4
 * for the outer loop): reverse-mode differentiation of the primal loop of
 * mlp_unit (use_ln = 1), token by token.  Per token, at the batch-start state
 * S: a = k W1 + c1, h = GELU(a), y = h W2 + c2, Delta2 = the LN+residual
 * backward at y (as in ln_residual_delta), m = Delta2 W2^T, d1 = m GELU'(a);
 * the updates use d1 and Delta2; the output is z = q + gamma LN(p) + beta with
 * p = GELU(q W1_t + c1_t) W2_t + c2_t at the state after the token.
 */
static void mlp_ln_unit_backward(int T, int d, int m, int b, const double *Q, const double *K, const double *V,
                                 const double *eta, const double *W1_0, const double *c1_0, const double *W2_0,
                                 const double *c2_0, const double *gamma, const double *beta, double eps,
                                 const double *dZ, const double *dW1o, const double *dc1o, const double *dW2o,
                                 const double *dc2o, double *dQ, double *dK, double *dV, double *deta, double *dW1,
                                 double *dc1, double *dW2, double *dc2, double *dgamma, double *dbeta) {
    const size_t n1 = (size_t)d * m;
    const int nb = (T + b - 1) / b;
    const size_t sz = n1 + m + n1 + d;   /* one state: W1, c1, W2, c2 */
    double *starts = malloc((size_t)(nb > 0 ? nb : 1) * sz * sizeof(double));
    double *run = malloc((size_t)(b + 1) * sz * sizeof(double));
    double *cur = malloc(sz * sizeof(double));
    double *D = malloc(sz * sizeof(double)), *Ds = malloc(sz * sizeof(double));
    /* per token of a batch */
    double *A = malloc((size_t)b * m * sizeof(double)), *Hh = malloc((size_t)b * m * sizeof(double));
    double *Mm = malloc((size_t)b * m * sizeof(double)), *D1 = malloc((size_t)b * m * sizeof(double));
    double *XH = malloc((size_t)b * d * sizeof(double)), *EE = malloc((size_t)b * d * sizeof(double));
    double *UU = malloc((size_t)b * d * sizeof(double)), *D2 = malloc((size_t)b * d * sizeof(double));
    double *RR = malloc((size_t)b * sizeof(double)), *MGX = malloc((size_t)b * sizeof(double));
    double *y = malloc(d * sizeof(double)), *pp = malloc(d * sizeof(double)), *xo = malloc(d * sizeof(double));
    double *t1 = malloc(d * sizeof(double)), *dp = malloc(d * sizeof(double)), *dd2 = malloc(d * sizeof(double));
    double *du = malloc(d * sizeof(double)), *dxh = malloc(d * sizeof(double)), *dy = malloc(d * sizeof(double));
    double *aq = malloc(m * sizeof(double)), *hq = malloc(m * sizeof(double)), *daq = malloc(m * sizeof(double));
    double *dd1 = malloc(m * sizeof(double)), *dm = malloc(m * sizeof(double)), *dh = malloc(m * sizeof(double));
    double *da = malloc(m * sizeof(double));
    #define W1P(x) (x)
    #define C1P(x) ((x) + n1)
    #define W2P(x) ((x) + n1 + m)
    #define C2P(x) ((x) + n1 + m + n1)

    /* token i of the batch at the batch-start state S: a, h, the LN quantities, Delta2, m, d1 */
    #define BATCH_FWD(t, i, S)                                                                         \
        do {                                                                                           \
            const double *k_ = K + (size_t)(t) * d, *v_ = V + (size_t)(t) * d;                         \
            double *a_ = A + (size_t)(i) * m, *h_ = Hh + (size_t)(i) * m;                              \
            double *x_ = XH + (size_t)(i) * d, *e_ = EE + (size_t)(i) * d;                             \
            double *u_ = UU + (size_t)(i) * d, *d2_ = D2 + (size_t)(i) * d;                            \
            vec_mat(d, m, k_, W1P(S), a_);                                                             \
            for (int p = 0; p < m; ++p) { a_[p] += C1P(S)[p]; h_[p] = gelu(a_[p]); }                   \
            vec_mat(m, d, h_, W2P(S), y);                                                              \
            for (int j = 0; j < d; ++j) y[j] += C2P(S)[j];                                             \
            RR[i] = layer_norm(d, y, eps, x_);                                                         \
            double mg = 0.0, mgx_ = 0.0;                                                               \
            for (int j = 0; j < d; ++j) {                                                              \
                e_[j] = k_[j] + gamma[j] * x_[j] + beta[j] - v_[j];                                    \
                mg += gamma[j] * e_[j];                                                                \
                mgx_ += gamma[j] * e_[j] * x_[j];                                                      \
            }                                                                                          \
            mg /= d;                                                                                   \
            mgx_ /= d;                                                                                 \
            MGX[i] = mgx_;                                                                             \
            for (int j = 0; j < d; ++j) {                                                              \
                u_[j] = gamma[j] * e_[j] - mg - x_[j] * mgx_;                                          \
                d2_[j] = RR[i] * u_[j];                                                                \
            }                                                                                          \
            for (int p = 0; p < m; ++p) {                                                              \
                double acc = 0.0;                                                                      \
                for (int j = 0; j < d; ++j) acc += W2P(S)[(size_t)p * d + j] * d2_[j];                 \
                Mm[(size_t)(i) * m + p] = acc;                                                         \
                D1[(size_t)(i) * m + p] = acc * gelu_grad(a_[p]);                                      \
            }                                                                                          \
        } while (0)
    /* one token's update applied to state X (in place) */
    #define TOKEN_UPD(t, i, X)                                                                         \
        do {                                                                                           \
            const double *k_ = K + (size_t)(t) * d, et_ = eta[t];                                      \
            const double *d1_ = D1 + (size_t)(i) * m, *h_ = Hh + (size_t)(i) * m;                      \
            const double *d2_ = D2 + (size_t)(i) * d;                                                  \
            for (int a2 = 0; a2 < d; ++a2)                                                             \
                for (int p = 0; p < m; ++p) W1P(X)[(size_t)a2 * m + p] -= et_ * k_[a2] * d1_[p];       \
            for (int p = 0; p < m; ++p) C1P(X)[p] -= et_ * d1_[p];                                     \
            for (int p = 0; p < m; ++p)                                                                \
                for (int j = 0; j < d; ++j) W2P(X)[(size_t)p * d + j] -= et_ * h_[p] * d2_[j];         \
            for (int j = 0; j < d; ++j) C2P(X)[j] -= et_ * d2_[j];                                     \
        } while (0)

    memcpy(W1P(cur), W1_0, n1 * sizeof(double));
    if (c1_0) memcpy(C1P(cur), c1_0, m * sizeof(double)); else memset(C1P(cur), 0, m * sizeof(double));
    memcpy(W2P(cur), W2_0, n1 * sizeof(double));
    if (c2_0) memcpy(C2P(cur), c2_0, d * sizeof(double)); else memset(C2P(cur), 0, d * sizeof(double));
    for (int i = 0; i < nb; ++i) {
        const int t0 = i * b, t1_ = (t0 + b < T) ? t0 + b : T;
        memcpy(starts + (size_t)i * sz, cur, sz * sizeof(double));
        for (int t = t0; t < t1_; ++t) BATCH_FWD(t, t - t0, starts + (size_t)i * sz);
        for (int t = t0; t < t1_; ++t) TOKEN_UPD(t, t - t0, cur);
    }
    memset(D, 0, sz * sizeof(double));
    if (dW1o) memcpy(W1P(D), dW1o, n1 * sizeof(double));
    if (dc1o) memcpy(C1P(D), dc1o, m * sizeof(double));
    if (dW2o) memcpy(W2P(D), dW2o, n1 * sizeof(double));
    if (dc2o) memcpy(C2P(D), dc2o, d * sizeof(double));
    memset(dgamma, 0, d * sizeof(double));
    memset(dbeta, 0, d * sizeof(double));
    for (int i = nb - 1; i >= 0; --i) {
        const int t0 = i * b, t1_ = (t0 + b < T) ? t0 + b : T;
        const double *S = starts + (size_t)i * sz;
        for (int t = t0; t < t1_; ++t) BATCH_FWD(t, t - t0, S);
        memcpy(run, S, sz * sizeof(double));
        for (int t = t0; t < t1_; ++t) {
            memcpy(run + (size_t)(t - t0 + 1) * sz, run + (size_t)(t - t0) * sz, sz * sizeof(double));
            TOKEN_UPD(t, t - t0, run + (size_t)(t - t0 + 1) * sz);
        }
        memset(Ds, 0, sz * sizeof(double));
        for (int t = t1_ - 1; t >= t0; --t) {
            const int li = t - t0;
            const double *q = Q + (size_t)t * d, *k = K + (size_t)t * d;
            const double *Rt = run + (size_t)(li + 1) * sz;   /* state after token t */
            const double *a = A + (size_t)li * m, *h = Hh + (size_t)li * m, *mm = Mm + (size_t)li * m;
            const double *d1 = D1 + (size_t)li * m;
            const double *xh = XH + (size_t)li * d, *e = EE + (size_t)li * d, *u = UU + (size_t)li * d;
            const double *d2 = D2 + (size_t)li * d;
            double *dq = dQ + (size_t)t * d, *dk = dK + (size_t)t * d, *dv = dV + (size_t)t * d;
            for (int j = 0; j < d; ++j) { dq[j] = 0.0; dk[j] = 0.0; }
            /* z = q + gamma LN(p) + beta, p = GELU(q W1_t + c1_t) W2_t + c2_t */
            if (dZ) {
                const double *dz = dZ + (size_t)t * d;
                vec_mat(d, m, q, W1P(Rt), aq);
                for (int p = 0; p < m; ++p) { aq[p] += C1P(Rt)[p]; hq[p] = gelu(aq[p]); }
                vec_mat(m, d, hq, W2P(Rt), pp);
                for (int j = 0; j < d; ++j) pp[j] += C2P(Rt)[j];
                const double ro = layer_norm(d, pp, eps, xo);
                for (int j = 0; j < d; ++j) {
                    dq[j] += dz[j];
                    dgamma[j] += dz[j] * xo[j];
                    dbeta[j] += dz[j];
                    t1[j] = gamma[j] * dz[j];
                }
                ln_adjoint(d, xo, ro, t1, dp);
                for (int p = 0; p < m; ++p) {
                    double acc = 0.0;
                    for (int j = 0; j < d; ++j) acc += dp[j] * W2P(Rt)[(size_t)p * d + j];
                    daq[p] = acc * gelu_grad(aq[p]);
                }
                for (int p = 0; p < m; ++p)
                    for (int j = 0; j < d; ++j) W2P(D)[(size_t)p * d + j] += hq[p] * dp[j];
                for (int j = 0; j < d; ++j) C2P(D)[j] += dp[j];
                for (int a2 = 0; a2 < d; ++a2) {
                    double acc = 0.0;
                    for (int p = 0; p < m; ++p) acc += daq[p] * W1P(Rt)[(size_t)a2 * m + p];
                    dq[a2] += acc;
                }
                for (int a2 = 0; a2 < d; ++a2)
                    for (int p = 0; p < m; ++p) W1P(D)[(size_t)a2 * m + p] += q[a2] * daq[p];
                for (int p = 0; p < m; ++p) C1P(D)[p] += daq[p];
            }
            /* the token's update: W1 -= eta k^T d1, c1 -= eta d1, W2 -= eta h^T Delta2, c2 -= eta Delta2 */
            double g = 0.0;
            for (int p = 0; p < m; ++p) {
                double acc = C1P(D)[p];
                for (int a2 = 0; a2 < d; ++a2) acc += k[a2] * W1P(D)[(size_t)a2 * m + p];
                dd1[p] = -eta[t] * acc;
                g += acc * d1[p];
            }
            for (int j = 0; j < d; ++j) {
                double acc = C2P(D)[j];
                for (int p = 0; p < m; ++p) acc += h[p] * W2P(D)[(size_t)p * d + j];
                dd2[j] = -eta[t] * acc;
                g += acc * d2[j];
            }
            deta[t] = -g;
            for (int a2 = 0; a2 < d; ++a2) {
                double acc = 0.0;
                for (int p = 0; p < m; ++p) acc += d1[p] * W1P(D)[(size_t)a2 * m + p];
                dk[a2] += -eta[t] * acc;
            }
            for (int p = 0; p < m; ++p) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += d2[j] * W2P(D)[(size_t)p * d + j];
                dh[p] = -eta[t] * acc;
            }
            /* d1 = m GELU'(a), m = Delta2 W2s^T */
            for (int p = 0; p < m; ++p) {
                dm[p] = dd1[p] * gelu_grad(a[p]);
                da[p] = dd1[p] * mm[p] * gelu_grad2(a[p]);
            }
            for (int j = 0; j < d; ++j) {
                double acc = 0.0;
                for (int p = 0; p < m; ++p) acc += dm[p] * W2P(S)[(size_t)p * d + j];
                dd2[j] += acc;
            }
            for (int p = 0; p < m; ++p)
                for (int j = 0; j < d; ++j) W2P(Ds)[(size_t)p * d + j] += dm[p] * d2[j];
            /* Delta2 = r u, u = g - mean(g) - xh mean(g xh), g = gamma e, e = k + gamma xh + beta - v */
            double dr = 0.0;
            for (int j = 0; j < d; ++j) { dr += dd2[j] * u[j]; du[j] = RR[li] * dd2[j]; }
            double mdu = 0.0, mdux = 0.0;
            for (int j = 0; j < d; ++j) { mdu += du[j]; mdux += du[j] * xh[j]; }
            mdu /= d;
            mdux /= d;
            for (int j = 0; j < d; ++j) {
                const double dg = du[j] - mdu - xh[j] * mdux;
                const double de = gamma[j] * dg;
                dxh[j] = -du[j] * MGX[li] - gamma[j] * e[j] * mdux + gamma[j] * de;
                dgamma[j] += e[j] * dg + xh[j] * de;
                dbeta[j] += de;
                dk[j] += de;
                dv[j] = -de;
            }
            /* xh = LN(y) and the r of Delta2 = r u */
            ln_adjoint(d, xh, RR[li], dxh, dy);
            for (int j = 0; j < d; ++j) dy[j] += dr * (-RR[li] * RR[li] * xh[j] / d);
            /* y = h W2s + c2s */
            for (int p = 0; p < m; ++p) {
                double acc = 0.0;
                for (int j = 0; j < d; ++j) acc += dy[j] * W2P(S)[(size_t)p * d + j];
                dh[p] += acc;
            }
            for (int p = 0; p < m; ++p)
                for (int j = 0; j < d; ++j) W2P(Ds)[(size_t)p * d + j] += h[p] * dy[j];
            for (int j = 0; j < d; ++j) C2P(Ds)[j] += dy[j];
            /* h = GELU(a), a = k W1s + c1s */
            for (int p = 0; p < m; ++p) da[p] += dh[p] * gelu_grad(a[p]);
            for (int a2 = 0; a2 < d; ++a2) {
                double acc = 0.0;
                for (int p = 0; p < m; ++p) acc += da[p] * W1P(S)[(size_t)a2 * m + p];
                dk[a2] += acc;
            }
            for (int a2 = 0; a2 < d; ++a2)
                for (int p = 0; p < m; ++p) W1P(Ds)[(size_t)a2 * m + p] += k[a2] * da[p];
            for (int p = 0; p < m; ++p) C1P(Ds)[p] += da[p];
        }
        for (size_t x = 0; x < sz; ++x) D[x] += Ds[x];
    }
    #undef BATCH_FWD
    #undef TOKEN_UPD
    memcpy(dW1, W1P(D), n1 * sizeof(double));
    memcpy(dc1, C1P(D), m * sizeof(double));
    memcpy(dW2, W2P(D), n1 * sizeof(double));
    memcpy(dc2, C2P(D), d * sizeof(double));
    #undef W1P
    #undef C1P
    #undef W2P
    #undef C2P
    free(starts); free(run); free(cur); free(D); free(Ds); free(A); free(Hh); free(Mm); free(D1);
    free(XH); free(EE); free(UU); free(D2); free(RR); free(MGX); free(y); free(pp); free(xo); free(t1); free(dp);
    free(dd2); free(du); free(dxh); free(dy); free(aq); free(hq); free(daq); free(dd1); free(dm); free(dh); free(da);
}

int ttt_oracle_mlp_ln_backward(int B, int H, int T, int d, int m, int b, const double *Q, const double *K,
                               const double *V, const double *eta, const double *W1, const double *c1,
                               const double *W2, const double *c2, long long p_bstride_scale, const double *gamma,
                               const double *beta, double eps, const double *dZ, const double *dW1o,
                               const double *dc1o, const double *dW2o, const double *dc2o, double *dQ, double *dK,
                               double *dV, double *deta, double *dW1, double *dc1, double *dW2, double *dc2,
                               double *dgamma, double *dbeta, int nthreads) {
    if (B < 0 || H < 0 || T < 0 || d <= 0 || m <= 0 || b <= 0 || !Q || !K || !V || !eta || !W1 || !W2 ||
        !gamma || !beta || !(eps > 0.0) || !dQ || !dK || !dV || !deta || !dW1 || !dc1 || !dW2 || !dc2 ||
        !dgamma || !dbeta)
        return 1;
    const long long units = (long long)B * H;
#ifdef _OPENMP
    if (nthreads > 0) omp_set_num_threads(nthreads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long long u = 0; u < units; ++u) {
        const long long pu = p_bstride_scale ? u : (u % H);
        const long long hd = u % H;
        const size_t tok = (size_t)u * T * d;
        mlp_ln_unit_backward(T, d, m, b, Q + tok, K + tok, V + tok, eta + (size_t)u * T, W1 + (size_t)pu * d * m,
                             c1 ? c1 + (size_t)pu * m : NULL, W2 + (size_t)pu * m * d,
                             c2 ? c2 + (size_t)pu * d : NULL, gamma + (size_t)hd * d, beta + (size_t)hd * d, eps,
                             dZ ? dZ + tok : NULL, dW1o ? dW1o + (size_t)u * d * m : NULL,
                             dc1o ? dc1o + (size_t)u * m : NULL, dW2o ? dW2o + (size_t)u * m * d : NULL,
                             dc2o ? dc2o + (size_t)u * d : NULL, dQ + tok, dK + tok, dV + tok, deta + (size_t)u * T,
                             dW1 + (size_t)u * d * m, dc1 + (size_t)u * m, dW2 + (size_t)u * m * d,
                             dc2 + (size_t)u * d, dgamma + (size_t)u * d, dbeta + (size_t)u * d);
    }
    (void)nthreads;
    return 0;
}

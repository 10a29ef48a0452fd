/*
 * Oracle for the Titans neural long-term memory -- TEST INFRASTRUCTURE ONLY.
 *
 * Only tests/, the smoke check and bench.py's CPU-baseline leg may load this
 * code. The product path (the CUDA library) never calls it, and this file
 * shares no code, header or constant with the CUDA path.
 *
 * It runs the memory's defining recurrence token by token, in fp64, on inputs
 * that were already rounded to the GPU input dtype (bf16 values are exact in
 * the float32 arrays passed here). Sources, all from the pages on
 * "Titans: Learning to Memorize at Test Time":
 *
 *  - loss:       l(M; x_t) = || M(k_t) - v_t ||_2^2       (walk-through, sec. 3.1 "Objective")
 *  - momentum:   S_t = eta_t S_{t-1} - theta_t grad l      (sec. 3.1 "Learning Process and
 *                                                           Surprise Metric"; German summary,
 *                                                           "Verbesserte Aktualisierungsregel")
 *  - forgetting: M_t = (1 - alpha_t) M_{t-1} + S_t         (sec. 3.1 "Forgetting Mechanism")
 *  - memory:     linear M(k) = W k (sec. 3.1 "Memory Architecture");
 *                MLP M(x) = W2 sigma(W1 x), sigma = SiLU   (hotdry blog sec. 3.1; SiLU per the
 *                                                           architecture notes, sec. 4.4)
 *  - retrieval:  y_t = M*(q_t), a forward pass with no weight change (sec. 3.1 "Retrieving a Memory")
 *  - chunking:   every token of a chunk takes its gradient at the weights the chunk started
 *                with, t' = t - mod(t, b)                  (sec. 3.2 "How to Parallelize ...")
 *
 * Readings where the pages are silent or garbled (each listed in the design notes):
 *  - the gradient is the exact derivative of the squared l2 loss (factor 2 kept);
 *  - tokens of chunk c see the state left by the last token of chunk c-1 (0-based chunks);
 *  - retrieval of every token of chunk c uses those chunk-start weights;
 *  - a last chunk shorter than b follows the same rules;
 *  - the MLP has no bias, residual or norm inside it.
 *
 * Layouts (row-major, one "unit" = one (batch, head) pair):
 *   k, q, v      [units][T][d]  float (values already rounded to the input dtype)
 *   alpha,eta,theta [units][T]  float
 *   MLP:    W1, S1 [units][h][d], W2, S2 [units][d][h]   double, read and overwritten
 *   linear: W1 = W, S1 = S [units][d][d] (W2, S2 unused)   double, read and overwritten
 *   y       [units][T][d]  double, or NULL to skip retrieval output
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

static double sigmoid(double z) { return 1.0 / (1.0 + exp(-z)); }

/* Linear memory: out = W x, W is [d][d] (rows = output features). */
static void linear_apply(int d, const double *W, const double *x, double *out) {
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int m = 0; m < d; ++m) s += W[(size_t)i * d + m] * x[m];
        out[i] = s;
    }
}

/* MLP memory: z = W1 x (h), a = z * sigmoid(z), out = W2 a (d). */
static void mlp_apply(int d, int h, const double *W1, const double *W2, const double *x,
                      double *z, double *a, double *out) {
    for (int j = 0; j < h; ++j) {
        double s = 0.0;
        for (int m = 0; m < d; ++m) s += W1[(size_t)j * d + m] * x[m];
        z[j] = s;
        a[j] = s * sigmoid(s);
    }
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < h; ++j) s += W2[(size_t)i * h + j] * a[j];
        out[i] = s;
    }
}

/*
 * Gradient of || W2 silu(W1 k) - v ||^2 with respect to W1 and W2, by the chain rule:
 *   e = W2 a - v,  dl/dout = 2 e
 *   dl/dW2[i][j] = 2 e_i a_j
 *   dl/da_j      = sum_i W2[i][j] 2 e_i
 *   da/dz        = silu'(z) = s (1 + z (1 - s)),  s = sigmoid(z)
 *   dl/dW1[j][m] = dl/da_j * silu'(z_j) * k_m
 */
static void mlp_grad(int d, int h, const double *W1, const double *W2, const double *k,
                     const double *v, double *z, double *a, double *out, double *ge,
                     double *delta, double *gW1, double *gW2) {
    mlp_apply(d, h, W1, W2, k, z, a, out);
    for (int i = 0; i < d; ++i) ge[i] = 2.0 * (out[i] - v[i]);
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < h; ++j) gW2[(size_t)i * h + j] = ge[i] * a[j];
    for (int j = 0; j < h; ++j) {
        double back = 0.0;
        for (int i = 0; i < d; ++i) back += W2[(size_t)i * h + j] * ge[i];
        double s = sigmoid(z[j]);
        delta[j] = back * s * (1.0 + z[j] * (1.0 - s));
    }
    for (int j = 0; j < h; ++j)
        for (int m = 0; m < d; ++m) gW1[(size_t)j * d + m] = delta[j] * k[m];
}

/* Gradient of || W k - v ||^2 with respect to W: 2 (W k - v) k^T. */
static void linear_grad(int d, const double *W, const double *k, const double *v,
                        double *out, double *gW) {
    linear_apply(d, W, k, out);
    for (int i = 0; i < d; ++i) {
        double e2 = 2.0 * (out[i] - v[i]);
        for (int m = 0; m < d; ++m) gW[(size_t)i * d + m] = e2 * k[m];
    }
}

/* S <- eta S - theta g ; W <- (1 - alpha) W + S   (momentum, then forgetting, new S in W) */
static void update(size_t n, double alpha, double eta, double theta, const double *g,
                   double *W, double *S) {
    for (size_t i = 0; i < n; ++i) {
        S[i] = eta * S[i] - theta * g[i];
        W[i] = (1.0 - alpha) * W[i] + S[i];
    }
}

static void load_row(int d, const float *src, double *dst) {
    for (int m = 0; m < d; ++m) dst[m] = (double)src[m];
}

static int run_unit(long T, int d, int h, int chunk, const float *k, const float *q,
                    const float *v, const float *alpha, const float *eta, const float *theta,
                    double *W1, double *W2, double *S1, double *S2, double *y) {
    const int linear = (h == 0);
    const size_t n1 = linear ? (size_t)d * d : (size_t)h * d;
    const size_t n2 = linear ? 0 : (size_t)d * h;
    const int hh = linear ? 1 : h;
    /* one allocation for all per-unit scratch */
    size_t need = 2 * (n1 + n2) /* chunk-start copies + gradients */ + 3 * (size_t)d + 4 * (size_t)hh + 2 * (size_t)d;
    double *buf = (double *)malloc(need * sizeof(double));
    if (!buf) return 1;
    double *W1bar = buf, *W2bar = W1bar + n1, *g1 = W2bar + n2, *g2 = g1 + n1;
    double *kx = g2 + n2, *vx = kx + d, *qx = vx + d;
    double *z = qx + d, *a = z + hh, *delta = a + hh, *zq = delta + hh;
    double *out = zq + hh, *ge = out + d;

    for (long t = 0; t < T; ++t) {
        if (t % chunk == 0) { /* chunk start: freeze the weights every token of the chunk uses */
            memcpy(W1bar, W1, n1 * sizeof(double));
            if (!linear) memcpy(W2bar, W2, n2 * sizeof(double));
        }
        load_row(d, k + (size_t)t * d, kx);
        load_row(d, v + (size_t)t * d, vx);
        load_row(d, q + (size_t)t * d, qx);
        if (y) { /* retrieval with the chunk-start weights, no update */
            double *yt = y + (size_t)t * d;
            if (linear) linear_apply(d, W1bar, qx, yt);
            else mlp_apply(d, h, W1bar, W2bar, qx, zq, a, yt);
        }
        if (linear) {
            linear_grad(d, W1bar, kx, vx, out, g1);
            update(n1, alpha[t], eta[t], theta[t], g1, W1, S1);
        } else {
            mlp_grad(d, h, W1bar, W2bar, kx, vx, z, a, out, ge, delta, g1, g2);
            update(n1, alpha[t], eta[t], theta[t], g1, W1, S1);
            update(n2, alpha[t], eta[t], theta[t], g2, W2, S2);
        }
    }
    free(buf);
    return 0;
}

/* Returns 0 on success, 1 on a bad argument or an allocation failure. */
int titans_oracle_forward(long units, long T, int d, int h, int chunk, const float *k,
                          const float *q, const float *v, const float *alpha, const float *eta,
                          const float *theta, double *W1, double *W2, double *S1, double *S2,
                          double *y, int n_threads) {
    if (units < 0 || T < 0 || d <= 0 || h < 0 || chunk <= 0) return 1;
    if (h > 0 && (!W2 || !S2)) return 1;
    const size_t n1 = h == 0 ? (size_t)d * d : (size_t)h * d;
    const size_t n2 = h == 0 ? 0 : (size_t)d * h;
    int err = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
    for (long u = 0; u < units; ++u) {
        err |= run_unit(T, d, h, chunk, k + (size_t)u * T * d, q + (size_t)u * T * d,
                        v + (size_t)u * T * d, alpha + (size_t)u * T, eta + (size_t)u * T,
                        theta + (size_t)u * T, W1 + u * n1, h ? W2 + u * n2 : NULL,
                        S1 + u * n1, h ? S2 + u * n2 : NULL, y ? y + (size_t)u * T * d : NULL);
    }
    (void)n_threads;
    return err;
}

/*
 * Deep memory (walk-through sec. 3.1 "Memory Architecture": an MLP with L_M >= 2 layers; sec. 5.5
 * "The Effect of Deep Memory"): M(x) = W_L silu(W_{L-1} ... silu(W_1 x)), every hidden layer h
 * wide, no bias. The L layers' weights of one unit are packed one after another, each row-major
 * [out][in]: W_1 [h][d], W_2 .. W_{L-1} [h][h], W_L [d][h].
 */
static size_t deep_size(int d, int h, int L) { return 2 * (size_t)h * d + (size_t)(L - 2) * h * h; }

static size_t deep_offset(int d, int h, int l) { /* start of layer l (0-based, l < L) */
    return l == 0 ? 0 : (size_t)h * d + (size_t)(l - 1) * h * h;
}

/* Forward of one input x: z[l] = W_l a[l-1] (a[-1] = x), a[l] = silu(z[l]) for the L-1 hidden
 * layers (z, a are [L-1][h]); out = W_L a[L-2] (d). */
static void deep_forward(int d, int h, int L, const double *W, const double *x, double *z, double *a,
                         double *out) {
    const double *in = x;
    int n_in = d;
    for (int l = 0; l < L - 1; ++l) {
        const double *Wl = W + deep_offset(d, h, l);
        for (int j = 0; j < h; ++j) {
            double s = 0.0;
            for (int m = 0; m < n_in; ++m) s += Wl[(size_t)j * n_in + m] * in[m];
            z[(size_t)l * h + j] = s;
            a[(size_t)l * h + j] = s * sigmoid(s);
        }
        in = a + (size_t)l * h;
        n_in = h;
    }
    const double *WL = W + deep_offset(d, h, L - 1);
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < h; ++j) s += WL[(size_t)i * h + j] * in[j];
        out[i] = s;
    }
}

/*
 * Gradient of || M(k) - v ||^2 with respect to every layer, by the chain rule from the output:
 *   e = 2 (out - v) is dl/d out; the output layer's gradient is e a[L-2]^T;
 *   delta = dl/dz[l] = (W_{l+1}^T dl/dz[l+1]) * silu'(z[l]), silu'(z) = s (1 + z (1 - s));
 *   layer l's gradient is delta (its input)^T, the input of layer 0 being k.
 * g has the packed layout of W; delta and back are scratch of h doubles each.
 */
static void deep_grad(int d, int h, int L, const double *W, const double *k, const double *v, double *z,
                      double *a, double *out, double *e, double *delta, double *back, double *g) {
    deep_forward(d, h, L, W, k, z, a, out);
    for (int i = 0; i < d; ++i) e[i] = 2.0 * (out[i] - v[i]);
    /* output layer */
    const double *WL = W + deep_offset(d, h, L - 1);
    double *gL = g + deep_offset(d, h, L - 1);
    const double *aL = a + (size_t)(L - 2) * h;
    for (int i = 0; i < d; ++i)
        for (int j = 0; j < h; ++j) gL[(size_t)i * h + j] = e[i] * aL[j];
    for (int j = 0; j < h; ++j) {
        double b = 0.0;
        for (int i = 0; i < d; ++i) b += WL[(size_t)i * h + j] * e[i];
        const double zz = z[(size_t)(L - 2) * h + j], s = sigmoid(zz);
        delta[j] = b * s * (1.0 + zz * (1.0 - s));
    }
    /* hidden layers, from the last to the first */
    for (int l = L - 2; l >= 0; --l) {
        const double *in = l == 0 ? k : a + (size_t)(l - 1) * h;
        const int n_in = l == 0 ? d : h;
        double *gl = g + deep_offset(d, h, l);
        for (int j = 0; j < h; ++j)
            for (int m = 0; m < n_in; ++m) gl[(size_t)j * n_in + m] = delta[j] * in[m];
        if (l > 0) {
            const double *Wl = W + deep_offset(d, h, l);
            for (int m = 0; m < h; ++m) {
                double b = 0.0;
                for (int j = 0; j < h; ++j) b += Wl[(size_t)j * h + m] * delta[j];
                const double zz = z[(size_t)(l - 1) * h + m], s = sigmoid(zz);
                back[m] = b * s * (1.0 + zz * (1.0 - s));
            }
            memcpy(delta, back, (size_t)h * sizeof(double));
        }
    }
}

static int run_unit_deep(long T, int d, int h, int L, int chunk, const float *k, const float *q,
                         const float *v, const float *alpha, const float *eta, const float *theta,
                         double *W, double *S, double *y) {
    const size_t P = deep_size(d, h, L);
    const size_t need = 2 * P + 3 * (size_t)d + 2 * (size_t)(L - 1) * h + 2 * (size_t)h + 2 * (size_t)d;
    double *buf = (double *)malloc(need * sizeof(double));
    if (!buf) return 1;
    double *Wbar = buf, *g = Wbar + P, *kx = g + P, *vx = kx + d, *qx = vx + d;
    double *z = qx + d, *a = z + (size_t)(L - 1) * h, *delta = a + (size_t)(L - 1) * h, *back = delta + h;
    double *out = back + h, *e = out + d;
    for (long t = 0; t < T; ++t) {
        if (t % chunk == 0) memcpy(Wbar, W, P * sizeof(double)); /* chunk-start weights */
        load_row(d, k + (size_t)t * d, kx);
        load_row(d, v + (size_t)t * d, vx);
        load_row(d, q + (size_t)t * d, qx);
        if (y) deep_forward(d, h, L, Wbar, qx, z, a, y + (size_t)t * d); /* retrieval, no update */
        deep_grad(d, h, L, Wbar, kx, vx, z, a, out, e, delta, back, g);
        update(P, alpha[t], eta[t], theta[t], g, W, S);
    }
    free(buf);
    return 0;
}

/* Deep memory forward; W, S: [units][deep_size] packed; returns 0, or 1 on a bad argument or an
 * allocation failure. */
int titans_oracle_forward_deep(long units, long T, int d, int h, int L, int chunk, const float *k,
                               const float *q, const float *v, const float *alpha, const float *eta,
                               const float *theta, double *W, double *S, double *y, int n_threads) {
    if (units < 0 || T < 0 || d <= 0 || h <= 0 || L < 2 || chunk <= 0 || !W || !S) return 1;
    const size_t P = deep_size(d, h, L);
    int err = 0;
#ifdef _OPENMP
    if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel for schedule(dynamic, 1) reduction(| : err)
#endif
    for (long u = 0; u < units; ++u) {
        err |= run_unit_deep(T, d, h, L, chunk, k + (size_t)u * T * d, q + (size_t)u * T * d,
                             v + (size_t)u * T * d, alpha + (size_t)u * T, eta + (size_t)u * T,
                             theta + (size_t)u * T, W + u * P, S + u * P, y ? y + (size_t)u * T * d : NULL);
    }
    (void)n_threads;
    return err;
}

int titans_oracle_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

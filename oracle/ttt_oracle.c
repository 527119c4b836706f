/*
 * Plain fp64 CPU oracle for the TTT-MLP layer scan.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path (the CUDA library,
 * its Python binding) may link, import or call this file; only the tests,
 * the smoke check and the CPU-baseline leg of the benchmark use it.  It
 * shares no code, header, table or helper with the CUDA path.
 *
 * What it computes (One-Minute Video Generation with Test-Time Training,
 * paper notes page, section "关键设计 / TTT-MLP 层"):
 *   - the hidden state of a head is a two-layer MLP
 *         f(u; W) = W2 * GELU(W1 * u),  W1: [m x d], W2: [d x m], m = 4 d,
 *     with erf-based GELU and no biases;
 *   - for every token the state takes one gradient-descent step on the
 *     self-supervised loss  l(W; x_t) = || f(theta_K x_t; W) - theta_V x_t ||^2
 *         W_t = W_{t-1} - eta * grad_W l(W_{t-1}; x_t);
 *   - the output token is z_t = f(theta_Q x_t; W_t), i.e. it is read with the
 *     state AFTER the update of token t.
 * Mini-batch variant (chunk of b tokens, b = 1 being the rule above): every
 * gradient of a chunk is taken at the state at the start of the chunk, W^c,
 * and token t of the chunk is read with the prefix state
 *         W_t = W^c - eta * sum_{s0 <= s <= t} grad l(W^c; x_s).
 * The next chunk starts from the state after its last token.  The reverse
 * direction walks the tokens from T-1 down to 0 and forms its chunks in that
 * walking order (the first reverse chunk holds the last b tokens).
 *
 * Everything here is a direct transcription of those definitions: no
 * blocking, no fusion, no reordering of the sums beyond the natural loops.
 * Build: gcc -O2 -fopenmp -shared -fPIC (no -ffast-math).
 */
#include <math.h>
#include <stdlib.h>
#include <string.h>

/* erf-based GELU: GELU(a) = a * Phi(a), Phi(a) = (1 + erf(a / sqrt 2)) / 2. */
double ttt_ref_gelu(double a) {
    return 0.5 * a * (1.0 + erf(a / sqrt(2.0)));
}

/* d GELU / da = Phi(a) + a * phi(a), phi the standard normal density. */
double ttt_ref_gelu_prime(double a) {
    const double Phi = 0.5 * (1.0 + erf(a / sqrt(2.0)));
    const double phi = exp(-0.5 * a * a) / sqrt(2.0 * M_PI);
    return Phi + a * phi;
}

/* f(u; W) = W2 GELU(W1 u).  a, g are [m] work/out buffers, y is [d]. */
static void mlp_forward(int d, int m, const double* W1, const double* W2,
                        const double* u, double* a, double* g, double* y) {
    for (int i = 0; i < m; ++i) {
        double acc = 0.0;
        for (int j = 0; j < d; ++j) acc += W1[(size_t)i * d + j] * u[j];
        a[i] = acc;
        g[i] = ttt_ref_gelu(acc);
    }
    for (int j = 0; j < d; ++j) {
        double acc = 0.0;
        for (int i = 0; i < m; ++i) acc += W2[(size_t)j * m + i] * g[i];
        y[j] = acc;
    }
}

/*
 * Loss l(W) = || W2 GELU(W1 k) - v ||^2 and its gradient by the chain rule:
 *   e = W2 g - v;  dl/dW2[j][i] = 2 e_j g_i;
 *   delta_i = (sum_j 2 e_j W2[j][i]) * GELU'(a_i);  dl/dW1[i][j] = delta_i k_j.
 * G1 is [m x d], G2 is [d x m]; either may be NULL (loss only).
 */
double ttt_ref_inner_loss_grad(int d, int m, const double* W1, const double* W2,
                               const double* k, const double* v,
                               double* G1, double* G2) {
    double* a = (double*)malloc(sizeof(double) * (size_t)m);
    double* g = (double*)malloc(sizeof(double) * (size_t)m);
    double* y = (double*)malloc(sizeof(double) * (size_t)d);
    double* e = (double*)malloc(sizeof(double) * (size_t)d);
    mlp_forward(d, m, W1, W2, k, a, g, y);
    double loss = 0.0;
    for (int j = 0; j < d; ++j) {
        e[j] = y[j] - v[j];
        loss += e[j] * e[j];
    }
    if (G2) {
        for (int j = 0; j < d; ++j)
            for (int i = 0; i < m; ++i) G2[(size_t)j * m + i] = 2.0 * e[j] * g[i];
    }
    if (G1) {
        for (int i = 0; i < m; ++i) {
            double back = 0.0;
            for (int j = 0; j < d; ++j) back += 2.0 * e[j] * W2[(size_t)j * m + i];
            const double delta = back * ttt_ref_gelu_prime(a[i]);
            for (int j = 0; j < d; ++j) G1[(size_t)i * d + j] = delta * k[j];
        }
    }
    free(a); free(g); free(y); free(e);
    return loss;
}

/* z = f(q; W) for one token. */
void ttt_ref_mlp_apply(int d, int m, const double* W1, const double* W2,
                       const double* u, double* z) {
    double* a = (double*)malloc(sizeof(double) * (size_t)m);
    double* g = (double*)malloc(sizeof(double) * (size_t)m);
    mlp_forward(d, m, W1, W2, u, a, g, z);
    free(a); free(g);
}

/*
 * The literal per-token rule, with no notion of a chunk:
 *   W_t = W_{t-1} - eta grad l(W_{t-1}; k_t, v_t);  z_t = f(q_t; W_t).
 * Q, K, V, Z are [T x d] row-major; W1 [m x d], W2 [d x m] hold W_0 on entry
 * and the state after the last token on return.  reverse != 0 walks t from
 * T-1 down to 0.
 */
void ttt_ref_scan_per_token(int T, int d, int m, int reverse, double eta,
                            const double* Q, const double* K, const double* V,
                            double* W1, double* W2, double* Z) {
    const size_t n1 = (size_t)m * d;
    double* G1 = (double*)malloc(sizeof(double) * n1);
    double* G2 = (double*)malloc(sizeof(double) * n1);
    for (int n = 0; n < T; ++n) {
        const int t = reverse ? (T - 1 - n) : n;
        ttt_ref_inner_loss_grad(d, m, W1, W2, K + (size_t)t * d, V + (size_t)t * d, G1, G2);
        for (size_t p = 0; p < n1; ++p) {
            W1[p] -= eta * G1[p];
            W2[p] -= eta * G2[p];
        }
        ttt_ref_mlp_apply(d, m, W1, W2, Q + (size_t)t * d, Z + (size_t)t * d);
    }
    free(G1); free(G2);
}

/*
 * Mini-batch scan in the primal form.  For each chunk of b consecutive tokens
 * (in walking order), every gradient is evaluated at the chunk-start state
 * Wc; the running state W accumulates -eta * gradient token by token.
 *   zmode 0 (prefix reading, the graded one): z_t = f(q_t; W_t), W_t the
 *           running state right after token t's gradient is applied;
 *   zmode 1 (chunk-end reading, kept only to show the two differ): every token
 *           of a chunk is read with the state after the chunk's last token.
 * Arguments as in ttt_ref_scan_per_token.
 */
void ttt_ref_scan_chunked(int T, int d, int m, int b, int reverse, int zmode, double eta,
                          const double* Q, const double* K, const double* V,
                          double* W1, double* W2, double* Z) {
    const size_t n1 = (size_t)m * d;
    double* W1c = (double*)malloc(sizeof(double) * n1);
    double* W2c = (double*)malloc(sizeof(double) * n1);
    double* G1 = (double*)malloc(sizeof(double) * n1);
    double* G2 = (double*)malloc(sizeof(double) * n1);
    for (int n0 = 0; n0 < T; n0 += b) {
        const int n1end = (n0 + b < T) ? (n0 + b) : T;
        memcpy(W1c, W1, sizeof(double) * n1);
        memcpy(W2c, W2, sizeof(double) * n1);
        for (int n = n0; n < n1end; ++n) {
            const int t = reverse ? (T - 1 - n) : n;
            ttt_ref_inner_loss_grad(d, m, W1c, W2c, K + (size_t)t * d, V + (size_t)t * d, G1, G2);
            for (size_t p = 0; p < n1; ++p) {
                W1[p] -= eta * G1[p];
                W2[p] -= eta * G2[p];
            }
            if (zmode == 0)
                ttt_ref_mlp_apply(d, m, W1, W2, Q + (size_t)t * d, Z + (size_t)t * d);
        }
        if (zmode != 0) {
            for (int n = n0; n < n1end; ++n) {
                const int t = reverse ? (T - 1 - n) : n;
                ttt_ref_mlp_apply(d, m, W1, W2, Q + (size_t)t * d, Z + (size_t)t * d);
            }
        }
    }
    free(W1c); free(W2c); free(G1); free(G2);
}

/*
 * H independent heads, one OpenMP task per head.  Per head h the streams are
 * Q + h*T*d etc. ([H x T x d] contiguous), the states W1 + h*m*d, W2 + h*d*m.
 * b == 1 runs the literal per-token rule.
 */
void ttt_ref_scan_heads(int H, int T, int d, int m, int b, int reverse, double eta,
                        const double* Q, const double* K, const double* V,
                        double* W1, double* W2, double* Z) {
    const size_t sT = (size_t)T * d, sW = (size_t)m * d;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        if (b == 1)
            ttt_ref_scan_per_token(T, d, m, reverse, eta, Q + h * sT, K + h * sT, V + h * sT,
                                   W1 + h * sW, W2 + h * sW, Z + h * sT);
        else
            ttt_ref_scan_chunked(T, d, m, b, reverse, 0, eta, Q + h * sT, K + h * sT, V + h * sT,
                                 W1 + h * sW, W2 + h * sW, Z + h * sT);
    }
}

#ifdef _OPENMP
#include <omp.h>
#endif

/* Number of OpenMP threads ttt_ref_scan_heads will use (1 without OpenMP). */
int ttt_ref_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ---------------------------------------------------------------- TTT-Linear
 * The linear variant of the layer (paper notes page, "实验关键数据 / 消融实验":
 * TTT-Linear, the same layer with a linear hidden state):
 *     f(u; W) = W u,  W: [d x d],
 * with the loss, the gradient step, the prefix reading inside a chunk, the
 * gate and the two directions exactly as for the MLP state above.  For the
 * loss l(W) = || W k - v ||^2 the gradient is grad_W = 2 (W k - v) k^T.
 */

/* l(W; k, v) and its gradient G [d x d] (row-major). */
double ttt_ref_linear_grad(int d, const double* W, const double* k, const double* v, double* G) {
    double loss = 0.0;
    for (int i = 0; i < d; ++i) {
        double e = -v[i];
        for (int j = 0; j < d; ++j) e += W[(size_t)i * d + j] * k[j];
        loss += e * e;
        for (int j = 0; j < d; ++j) G[(size_t)i * d + j] = 2.0 * e * k[j];
    }
    return loss;
}

/* z = W u. */
void ttt_ref_linear_apply(int d, const double* W, const double* u, double* z) {
    for (int i = 0; i < d; ++i) {
        double s = 0.0;
        for (int j = 0; j < d; ++j) s += W[(size_t)i * d + j] * u[j];
        z[i] = s;
    }
}

/* The per-token rule: W_t = W_{t-1} - eta grad l(W_{t-1}; x_t), z_t = W_t q_t. */
void ttt_ref_linear_scan_per_token(int T, int d, int reverse, double eta, const double* Q, const double* K,
                                   const double* V, double* W, double* Z) {
    const size_t n = (size_t)d * d;
    double* G = (double*)malloc(sizeof(double) * n);
    for (int s = 0; s < T; ++s) {
        const int t = reverse ? (T - 1 - s) : s;
        ttt_ref_linear_grad(d, W, K + (size_t)t * d, V + (size_t)t * d, G);
        for (size_t p = 0; p < n; ++p) W[p] -= eta * G[p];
        ttt_ref_linear_apply(d, W, Q + (size_t)t * d, Z + (size_t)t * d);
    }
    free(G);
}

/* Mini-batch form: gradients at the chunk-start state, prefix reading. */
void ttt_ref_linear_scan_chunked(int T, int d, int b, int reverse, double eta, const double* Q, const double* K,
                                 const double* V, double* W, double* Z) {
    const size_t n = (size_t)d * d;
    double* Wc = (double*)malloc(sizeof(double) * n);
    double* G = (double*)malloc(sizeof(double) * n);
    for (int s0 = 0; s0 < T; s0 += b) {
        const int s1 = (s0 + b < T) ? (s0 + b) : T;
        memcpy(Wc, W, sizeof(double) * n);
        for (int s = s0; s < s1; ++s) {
            const int t = reverse ? (T - 1 - s) : s;
            ttt_ref_linear_grad(d, Wc, K + (size_t)t * d, V + (size_t)t * d, G);
            for (size_t p = 0; p < n; ++p) W[p] -= eta * G[p];
            ttt_ref_linear_apply(d, W, Q + (size_t)t * d, Z + (size_t)t * d);
        }
    }
    free(Wc); free(G);
}

/* H independent heads ([H x T x d] streams, W [H x d x d]), one OpenMP task each. */
void ttt_ref_linear_scan_heads(int H, int T, int d, int b, int reverse, double eta, const double* Q,
                               const double* K, const double* V, double* W, double* Z) {
    const size_t sT = (size_t)T * d, sW = (size_t)d * d;
#pragma omp parallel for schedule(dynamic, 1)
    for (int h = 0; h < H; ++h) {
        if (b == 1)
            ttt_ref_linear_scan_per_token(T, d, reverse, eta, Q + h * sT, K + h * sT, V + h * sT, W + h * sW,
                                          Z + h * sT);
        else
            ttt_ref_linear_scan_chunked(T, d, b, reverse, eta, Q + h * sT, K + h * sT, V + h * sT, W + h * sW,
                                        Z + h * sT);
    }
}

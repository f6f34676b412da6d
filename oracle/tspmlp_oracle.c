/*
 * tspmlp_oracle.c -- plain, slow fp64 CPU oracle for the column-then-row
 * sharded transformer MLP.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product library links, loads or
 * calls this file; only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark do.  It shares no code, header, table or helper with the CUDA
 * path.
 *
 * What it computes (all arithmetic in IEEE fp64, inputs are fp64 arrays,
 * every sum taken in natural index order, no blocking or reordering):
 *
 *   plain MLP  Y = GeLU(X.A).B
 *       "Tensor Parallelism: Splitting the Math", section "Why the
 *       column-then-row split -- and what happens in attention".
 *       GeLU is the exact erf form GeLU(z) = z * Phi(z) (the pages never
 *       name a variant; the textbook definition is taken).
 *   gated MLP  Y = (SiLU(X.Wg) (*) (X.Wu)).Wd,  SiLU(g) = g * sigmoid(g)
 *       "Folding Tensor and Sequence Parallelism for Memory-Efficient
 *       Transformer Training & Inference", Abstract ("for gated MLPs").
 *   column split of A (and of Wg, Wu), row split of B (Wd); shard w owns the
 *       half-open column range [w*f/P, (w+1)*f/P)
 *       "Tensor Parallelism: Splitting the Math", steps 2-5 of
 *       "One transformer MLP, split across two GPUs".
 *   the sum of the per-shard partial outputs
 *       same page, step 6 ("partial results sum into the exact output").
 *   the folded tensor-and-sequence (TSP) schedule: sequence shard s meets
 *       weight shard (s+t) mod P at ring step t and accumulates locally
 *       "Folding Tensor and Sequence Parallelism ...", Abstract.
 *   the backward pass (the pages only say the backward repeats the forward
 *       pattern: "Tensor Parallelism: Splitting the Math", the paragraph
 *       that counts the traffic); the gradients below are the closed-form
 *       derivatives of the forward definition.
 *
 * Layout: every matrix is dense row-major.
 *   X[n][d], A = Wg[d][f], Wu[d][f], B = Wd[f][d], Y[n][d], dY[n][d].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_ACT_GELU 0
#define ORACLE_ACT_SWIGLU 1

/* Standard normal CDF Phi(z) = (1 + erf(z / sqrt 2)) / 2. */
static double std_normal_cdf(double z) { return 0.5 * (1.0 + erf(z / sqrt(2.0))); }

/* Standard normal density phi(z) = exp(-z^2/2) / sqrt(2 pi). */
static double std_normal_pdf(double z) { return exp(-0.5 * z * z) / sqrt(2.0 * M_PI); }

static double sigmoid(double g) { return 1.0 / (1.0 + exp(-g)); }

/* The activation of one hidden unit: GeLU(z) for the plain MLP (u unused),
 * SiLU(g) * u for the gated MLP. */
static double act_value(int act, double g, double u) {
    if (act == ORACLE_ACT_GELU) return g * std_normal_cdf(g);
    return g * sigmoid(g) * u;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Pre-activations of one token row for hidden units j in [j0, j1):
 *   g[j-j0] = sum_k x[k] * A[k][j]      (k = 0 .. d-1, in order)
 *   u[j-j0] = sum_k x[k] * Wu[k][j]     (gated MLP only)                 */
static void row_preactivations(const double* x, const double* A, const double* Wu, int act,
                               int64_t d, int64_t f, int64_t j0, int64_t j1, double* g,
                               double* u) {
    int64_t w = j1 - j0;
    for (int64_t j = 0; j < w; ++j) {
        g[j] = 0.0;
        u[j] = 0.0;
    }
    for (int64_t k = 0; k < d; ++k) {
        const double xk = x[k];
        const double* arow = A + k * f + j0;
        for (int64_t j = 0; j < w; ++j) g[j] += xk * arow[j];
        if (act == ORACLE_ACT_SWIGLU) {
            const double* urow = Wu + k * f + j0;
            for (int64_t j = 0; j < w; ++j) u[j] += xk * urow[j];
        }
    }
}

/* Partial output of one token row from hidden units [j0, j1):
 *   y[c] = sum_{j=j0}^{j1-1} h[j-j0] * B[j][c]   (j in order)             */
static void row_down_projection(const double* h, const double* B, int64_t d, int64_t j0,
                                int64_t j1, double* y) {
    for (int64_t c = 0; c < d; ++c) y[c] = 0.0;
    for (int64_t j = j0; j < j1; ++j) {
        const double hj = h[j - j0];
        const double* brow = B + j * d;
        for (int64_t c = 0; c < d; ++c) y[c] += hj * brow[c];
    }
}

/* One token row through the hidden units [j0, j1): returns the partial output
 * in y_part (length d) and, if h_out is not NULL, the hidden activations. */
static void row_block(const double* x, const double* A, const double* Wu, const double* B, int act,
                      int64_t d, int64_t f, int64_t j0, int64_t j1, double* g, double* u,
                      double* h, double* y_part) {
    row_preactivations(x, A, Wu, act, d, f, j0, j1, g, u);
    for (int64_t j = 0; j < j1 - j0; ++j) h[j] = act_value(act, g[j], u[j]);
    row_down_projection(h, B, d, j0, j1, y_part);
}

/* Unsharded MLP: Y = act(X.A).B over all f hidden units. */
int oracle_mlp_forward(const double* X, const double* A, const double* Wu, const double* B,
                       int64_t n, int64_t d, int64_t f, int act, double* Y) {
    if (n < 0 || d <= 0 || f <= 0) return 1;
    if (act != ORACLE_ACT_GELU && act != ORACLE_ACT_SWIGLU) return 1;
    int err = 0;
#pragma omp parallel
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)f);
        double* u = (double*)malloc(sizeof(double) * (size_t)f);
        double* h = (double*)malloc(sizeof(double) * (size_t)f);
        if (!g || !u || !h) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n; ++i)
                row_block(X + i * d, A, Wu, B, act, d, f, 0, f, g, u, h, Y + i * d);
        }
        free(g);
        free(u);
        free(h);
    }
    return err;
}

/* Hidden activations H = act(X.A), H[n][f]. */
int oracle_mlp_hidden(const double* X, const double* A, const double* Wu, int64_t n, int64_t d,
                      int64_t f, int act, double* H) {
    if (n < 0 || d <= 0 || f <= 0) return 1;
    if (act != ORACLE_ACT_GELU && act != ORACLE_ACT_SWIGLU) return 1;
    int err = 0;
#pragma omp parallel
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)f);
        double* u = (double*)malloc(sizeof(double) * (size_t)f);
        if (!g || !u) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n; ++i) {
                row_preactivations(X + i * d, A, Wu, act, d, f, 0, f, g, u);
                for (int64_t j = 0; j < f; ++j) H[i * f + j] = act_value(act, g[j], u[j]);
            }
        }
        free(g);
        free(u);
    }
    return err;
}

/* One weight shard w of P: its hidden block Hw = act(X.A_w) (n x f/P) and its
 * partial output Yw = Hw.B_w (n x d), A_w = columns [w f/P, (w+1) f/P) of A,
 * B_w = the same rows of B.  Either output may be NULL. */
int oracle_mlp_shard_partial(const double* X, const double* A, const double* Wu, const double* B,
                             int64_t n, int64_t d, int64_t f, int act, int P, int w, double* Hw,
                             double* Yw) {
    if (n < 0 || d <= 0 || f <= 0 || P <= 0 || f % P != 0 || w < 0 || w >= P) return 1;
    if (act != ORACLE_ACT_GELU && act != ORACLE_ACT_SWIGLU) return 1;
    const int64_t fs = f / P, j0 = (int64_t)w * fs, j1 = j0 + fs;
    int err = 0;
#pragma omp parallel
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)fs);
        double* u = (double*)malloc(sizeof(double) * (size_t)fs);
        double* h = (double*)malloc(sizeof(double) * (size_t)fs);
        double* y = (double*)malloc(sizeof(double) * (size_t)d);
        if (!g || !u || !h || !y) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n; ++i) {
                row_block(X + i * d, A, Wu, B, act, d, f, j0, j1, g, u, h, y);
                if (Hw) memcpy(Hw + i * fs, h, sizeof(double) * (size_t)fs);
                if (Yw) memcpy(Yw + i * d, y, sizeof(double) * (size_t)d);
            }
        }
        free(g);
        free(u);
        free(h);
        free(y);
    }
    return err;
}

/* Column-then-row sharded MLP: Y = sum over w in order[0..P-1] of
 * act(X.A_w).B_w, the partial outputs added one shard after another into a
 * zero-initialised accumulator.  order == NULL means 0, 1, ..., P-1. */
int oracle_mlp_sharded(const double* X, const double* A, const double* Wu, const double* B,
                       int64_t n, int64_t d, int64_t f, int act, int P, const int* order,
                       double* Y) {
    if (n < 0 || d <= 0 || f <= 0 || P <= 0 || f % P != 0) return 1;
    if (act != ORACLE_ACT_GELU && act != ORACLE_ACT_SWIGLU) return 1;
    if (order) {
        /* must be a permutation of 0..P-1 */
        char* seen = (char*)calloc((size_t)P, 1);
        if (!seen) return 2;
        for (int t = 0; t < P; ++t) {
            if (order[t] < 0 || order[t] >= P || seen[order[t]]) {
                free(seen);
                return 1;
            }
            seen[order[t]] = 1;
        }
        free(seen);
    }
    const int64_t fs = f / P;
    int err = 0;
#pragma omp parallel
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)fs);
        double* u = (double*)malloc(sizeof(double) * (size_t)fs);
        double* h = (double*)malloc(sizeof(double) * (size_t)fs);
        double* y = (double*)malloc(sizeof(double) * (size_t)d);
        if (!g || !u || !h || !y) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n; ++i) {
                double* yi = Y + i * d;
                for (int64_t c = 0; c < d; ++c) yi[c] = 0.0;
                for (int t = 0; t < P; ++t) {
                    const int w = order ? order[t] : t;
                    row_block(X + i * d, A, Wu, B, act, d, f, (int64_t)w * fs,
                              (int64_t)(w + 1) * fs, g, u, h, y);
                    for (int64_t c = 0; c < d; ++c) yi[c] += y[c];
                }
            }
        }
        free(g);
        free(u);
        free(h);
        free(y);
    }
    return err;
}

/* Folded tensor-and-sequence schedule.  Tokens are cut into P equal sequence
 * shards; sequence shard s holds tokens [s n/P, (s+1) n/P).  At ring step
 * t = 0 .. P-1 it meets weight shard w = (s + t) mod P and adds that shard's
 * partial output into its own accumulator.  reverse != 0 walks the ring the
 * other way, w = (s - t) mod P. */
int oracle_mlp_tsp(const double* X, const double* A, const double* Wu, const double* B, int64_t n,
                   int64_t d, int64_t f, int act, int P, int reverse, double* Y) {
    if (n < 0 || d <= 0 || f <= 0 || P <= 0 || f % P != 0 || n % P != 0) return 1;
    if (act != ORACLE_ACT_GELU && act != ORACLE_ACT_SWIGLU) return 1;
    const int64_t fs = f / P, ns = n / P;
    int err = 0;
#pragma omp parallel
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)fs);
        double* u = (double*)malloc(sizeof(double) * (size_t)fs);
        double* h = (double*)malloc(sizeof(double) * (size_t)fs);
        double* y = (double*)malloc(sizeof(double) * (size_t)d);
        if (!g || !u || !h || !y) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n; ++i) {
                const int s = (int)(i / ns);
                double* yi = Y + i * d;
                for (int64_t c = 0; c < d; ++c) yi[c] = 0.0;
                for (int t = 0; t < P; ++t) {
                    const int w = reverse ? ((s - t) % P + P) % P : (s + t) % P;
                    row_block(X + i * d, A, Wu, B, act, d, f, (int64_t)w * fs,
                              (int64_t)(w + 1) * fs, g, u, h, y);
                    for (int64_t c = 0; c < d; ++c) yi[c] += y[c];
                }
            }
        }
        free(g);
        free(u);
        free(h);
        free(y);
    }
    return err;
}

/* Backward pass of the MLP for an upstream gradient dY[n][d].
 *
 *   G = X.A, (U = X.Wu), dH = dY.B^T
 *   plain:  H = GeLU(G);           dG = dH * GeLU'(G),  GeLU'(z) = Phi(z) + z phi(z)
 *   gated:  H = SiLU(G) * U;       dU = dH * SiLU(G)
 *                                  dG = dH * U * SiLU'(G),
 *                                  SiLU'(g) = s(g) (1 + g (1 - s(g))), s = sigmoid
 *   dX  = dG.A^T (+ dU.Wu^T)
 *   dA  = X^T.dG,  dWu = X^T.dU,  dB = H^T.dY
 *
 * dWu (and Wu) are ignored for the plain MLP.  Any output may be NULL. */
int oracle_mlp_backward(const double* X, const double* A, const double* Wu, const double* B,
                        const double* dY, int64_t n, int64_t d, int64_t f, int act, double* dX,
                        double* dA, double* dWu, double* dB) {
    if (n <= 0 || d <= 0 || f <= 0) return 1;
    if (act != ORACLE_ACT_GELU && act != ORACLE_ACT_SWIGLU) return 1;
    const size_t nf = (size_t)n * (size_t)f;
    double* H = (double*)malloc(sizeof(double) * nf);
    double* dG = (double*)malloc(sizeof(double) * nf);
    double* dU = (double*)malloc(sizeof(double) * nf);
    if (!H || !dG || !dU) {
        free(H);
        free(dG);
        free(dU);
        return 2;
    }
    int err = 0;
    /* per-row: pre-activations, dH, and the elementwise backward */
#pragma omp parallel
    {
        double* g = (double*)malloc(sizeof(double) * (size_t)f);
        double* u = (double*)malloc(sizeof(double) * (size_t)f);
        if (!g || !u) {
#pragma omp atomic write
            err = 2;
        } else {
#pragma omp for schedule(dynamic, 1)
            for (int64_t i = 0; i < n; ++i) {
                row_preactivations(X + i * d, A, Wu, act, d, f, 0, f, g, u);
                const double* dyi = dY + i * d;
                for (int64_t j = 0; j < f; ++j) {
                    /* dH[i][j] = sum_c dY[i][c] * B[j][c] */
                    double dh = 0.0;
                    const double* brow = B + j * d;
                    for (int64_t c = 0; c < d; ++c) dh += dyi[c] * brow[c];
                    const double gj = g[j];
                    if (act == ORACLE_ACT_GELU) {
                        H[i * f + j] = gj * std_normal_cdf(gj);
                        dG[i * f + j] = dh * (std_normal_cdf(gj) + gj * std_normal_pdf(gj));
                        dU[i * f + j] = 0.0;
                    } else {
                        const double s = sigmoid(gj);
                        H[i * f + j] = gj * s * u[j];
                        dU[i * f + j] = dh * gj * s;
                        dG[i * f + j] = dh * u[j] * s * (1.0 + gj * (1.0 - s));
                    }
                }
            }
        }
        free(g);
        free(u);
    }
    if (err) {
        free(H);
        free(dG);
        free(dU);
        return err;
    }
    if (dX) {
        /* dX[i][k] = sum_j dG[i][j] A[k][j] (+ sum_j dU[i][j] Wu[k][j]) */
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t i = 0; i < n; ++i) {
            for (int64_t k = 0; k < d; ++k) {
                double s = 0.0;
                const double* arow = A + k * f;
                for (int64_t j = 0; j < f; ++j) s += dG[i * f + j] * arow[j];
                if (act == ORACLE_ACT_SWIGLU) {
                    const double* urow = Wu + k * f;
                    for (int64_t j = 0; j < f; ++j) s += dU[i * f + j] * urow[j];
                }
                dX[i * d + k] = s;
            }
        }
    }
    if (dA || (dWu && act == ORACLE_ACT_SWIGLU)) {
        /* dA[k][j] = sum_i X[i][k] dG[i][j];  dWu[k][j] = sum_i X[i][k] dU[i][j].
         * One row k at a time; every (k, j) sum runs over i = 0 .. n-1 in order. */
#pragma omp parallel
        {
            double* sa = (double*)malloc(sizeof(double) * (size_t)f);
            double* su = (double*)malloc(sizeof(double) * (size_t)f);
            if (!sa || !su) {
#pragma omp atomic write
                err = 2;
            } else {
#pragma omp for schedule(dynamic, 1)
                for (int64_t k = 0; k < d; ++k) {
                    for (int64_t j = 0; j < f; ++j) sa[j] = su[j] = 0.0;
                    for (int64_t i = 0; i < n; ++i) {
                        const double xik = X[i * d + k];
                        const double* dgi = dG + i * f;
                        const double* dui = dU + i * f;
                        for (int64_t j = 0; j < f; ++j) sa[j] += xik * dgi[j];
                        if (act == ORACLE_ACT_SWIGLU)
                            for (int64_t j = 0; j < f; ++j) su[j] += xik * dui[j];
                    }
                    if (dA) memcpy(dA + k * f, sa, sizeof(double) * (size_t)f);
                    if (dWu && act == ORACLE_ACT_SWIGLU)
                        memcpy(dWu + k * f, su, sizeof(double) * (size_t)f);
                }
            }
            free(sa);
            free(su);
        }
    }
    if (dB && !err) {
        /* dB[j][c] = sum_i H[i][j] dY[i][c]; one row j at a time, i in order. */
#pragma omp parallel for schedule(dynamic, 1)
        for (int64_t j = 0; j < f; ++j) {
            double* dbj = dB + j * d;
            for (int64_t c = 0; c < d; ++c) dbj[c] = 0.0;
            for (int64_t i = 0; i < n; ++i) {
                const double hij = H[i * f + j];
                const double* dyi = dY + i * d;
                for (int64_t c = 0; c < d; ++c) dbj[c] += hij * dyi[c];
            }
        }
    }
    free(H);
    free(dG);
    free(dU);
    return err;
}

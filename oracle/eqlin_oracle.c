/*
 * eqlin_oracle.c -- the CPU oracle for the EQ-Linear layer.
 *
 * TEST INFRASTRUCTURE ONLY. Nothing on the product path may call, link or
 * load this file; only the test suite, the smoke check and the benchmark's
 * CPU-baseline leg use it. It shares no code, header or table with the
 * CUDA library.
 *
 * What it computes is the plain definition of the layer, written out as
 * loops, in double precision:
 *
 *   "Flash EQ-Linear: Accelerating Equivariant Linear Layers via Group-wise
 *    Discrete Fourier Transform" (abstract): the EQ-Linear layer is a
 *   circular convolution along the group dimension composed with a linear
 *   transform along channels.  The technical summary of the same paper
 *   (section "Insight Central") describes the weight as a group-circulant
 *   matrix built by replicating and cyclically shifting one set of learnable
 *   parameters.  Written as an index formula, with x laid out [N, C'*T]
 *   (index c*T+t), W laid out [D', C', T] and a bias b[D'] shared by the T
 *   group positions of an output channel:
 *
 *     y[n, d*T+s] = b[d] + sum_c sum_t W[d, c, (s-t) mod T] * x[n, c*T+t]
 *
 * The paper says the method is an exact acceleration (summary, "Garantias
 * Teoricas"), so the oracle is this definition and not the Fourier
 * algorithm.  The pages print no backward formulas; the backward functions
 * below are the exact derivatives of the forward definition above:
 *
 *     dx[n, c*T+t] = sum_d sum_s W[d, c, (s-t) mod T] * gy[n, d*T+s]
 *     dW[d, c, tau] = sum_n sum_s gy[n, d*T+s] * x[n, c*T + (s-tau) mod T]
 *     db[d]         = sum_n sum_s gy[n, d*T+s]
 *
 * Inputs are the already-rounded values of whatever precision the caller
 * uses, converted to double; every sum accumulates in double in the order
 * the loops state.  There is no blocking, no reordering and no transform.
 *
 * Each function optionally works on a subset: `rows` (token indices) for
 * forward/dx and `pairs` ((d, c) index pairs) for dW, so that full-size
 * workloads can be checked on sampled outputs.
 */
#include <stdint.h>
#ifdef _OPENMP
#include <omp.h>
#endif

static int64_t wrap(int64_t a, int64_t T)
{
    int64_t r = a % T;
    return r < 0 ? r + T : r;
}

int eqlin_oracle_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * y[i, d*T+s] for i in [0, n_out): token n = rows ? rows[i] : i.
 * x is [N_total, Cp*T]; y is [n_out, Dp*T]; b may be NULL (no bias).
 */
void eqlin_oracle_forward(int64_t T, int64_t Cp, int64_t Dp,
                          const double *x, const double *W, const double *b,
                          const int64_t *rows, int64_t n_out, double *y)
{
    int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < n_out; ++i) {
        const int64_t n = rows ? rows[i] : i;
        for (int64_t d = 0; d < Dp; ++d) {
            for (int64_t s = 0; s < T; ++s) {
                double acc = 0.0;
                for (int64_t c = 0; c < Cp; ++c)
                    for (int64_t t = 0; t < T; ++t)
                        acc += W[(d * Cp + c) * T + wrap(s - t, T)] *
                               x[n * Cp * T + c * T + t];
                y[i * Dp * T + d * T + s] = (b ? b[d] : 0.0) + acc;
            }
        }
    }
}

/*
 * dx[i, c*T+t] for i in [0, n_out): token n = rows ? rows[i] : i.
 * gy is [N_total, Dp*T]; dx is [n_out, Cp*T].
 */
void eqlin_oracle_backward_dx(int64_t T, int64_t Cp, int64_t Dp,
                              const double *gy, const double *W,
                              const int64_t *rows, int64_t n_out, double *dx)
{
    int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < n_out; ++i) {
        const int64_t n = rows ? rows[i] : i;
        for (int64_t c = 0; c < Cp; ++c) {
            for (int64_t t = 0; t < T; ++t) {
                double acc = 0.0;
                for (int64_t d = 0; d < Dp; ++d)
                    for (int64_t s = 0; s < T; ++s)
                        acc += W[(d * Cp + c) * T + wrap(s - t, T)] *
                               gy[n * Dp * T + d * T + s];
                dx[i * Cp * T + c * T + t] = acc;
            }
        }
    }
}

/*
 * dW over all N tokens.  If pairs is NULL, dW is the full [Dp, Cp, T] array
 * and n_pairs is ignored; otherwise pairs holds n_pairs (d, c) index pairs
 * and dW is [n_pairs, T].  db (length Dp) is written when not NULL.
 */
void eqlin_oracle_backward_dw(int64_t T, int64_t Cp, int64_t Dp, int64_t N,
                              const double *x, const double *gy,
                              const int64_t *pairs, int64_t n_pairs,
                              double *dW, double *db)
{
    const int64_t n_work = pairs ? n_pairs : Dp * Cp;
    int64_t j;
#pragma omp parallel for schedule(dynamic, 1)
    for (j = 0; j < n_work; ++j) {
        const int64_t d = pairs ? pairs[2 * j] : j / Cp;
        const int64_t c = pairs ? pairs[2 * j + 1] : j % Cp;
        for (int64_t tau = 0; tau < T; ++tau) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
                for (int64_t s = 0; s < T; ++s)
                    acc += gy[n * Dp * T + d * T + s] *
                           x[n * Cp * T + c * T + wrap(s - tau, T)];
            dW[j * T + tau] = acc;
        }
    }
    if (db) {
        int64_t d;
#pragma omp parallel for schedule(static)
        for (d = 0; d < Dp; ++d) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
                for (int64_t s = 0; s < T; ++s)
                    acc += gy[n * Dp * T + d * T + s];
            db[d] = acc;
        }
    }
}

/*
 * The same layer over any finite group G of order n given by its
 * multiplication table, for the reflection (dihedral) groups the paper names
 * as future work (technical summary, section "Limitacoes e Trabalho Futuro")
 * and which it does not spell out.  The plainest generalisation of the
 * cyclic formula above -- whose kernel index (s - t) mod T is h^-1 g for the
 * group elements g = s, h = t of Z_T -- is the group convolution
 *
 *     y[n, d*n+g]  = b[d] + sum_c sum_h W[d, c, h^-1 g] * x[n, c*n+h]
 *
 * which commutes with the left action (L_u x)[h] = x[u^-1 h] of every u in G.
 * Its exact gradients (derived from this definition):
 *
 *     dx[n, c*n+h] = sum_d sum_g W[d, c, h^-1 g] * gy[n, d*n+g]
 *     dW[d, c, u]  = sum_n sum_h x[n, c*n+h] * gy[n, d*n + h u]
 *     db[d]        = sum_n sum_g gy[n, d*n+g]
 *
 * mul[g*n + h] is the index of the product g h and inv[g] that of g^-1.
 */
void eqlin_oracle_forward_group(int64_t G, const int64_t *mul, const int64_t *inv,
                                int64_t Cp, int64_t Dp,
                                const double *x, const double *W, const double *b,
                                const int64_t *rows, int64_t n_out, double *y)
{
    int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < n_out; ++i) {
        const int64_t n = rows ? rows[i] : i;
        for (int64_t d = 0; d < Dp; ++d) {
            for (int64_t g = 0; g < G; ++g) {
                double acc = 0.0;
                for (int64_t c = 0; c < Cp; ++c)
                    for (int64_t h = 0; h < G; ++h)
                        acc += W[(d * Cp + c) * G + mul[inv[h] * G + g]] *
                               x[n * Cp * G + c * G + h];
                y[i * Dp * G + d * G + g] = (b ? b[d] : 0.0) + acc;
            }
        }
    }
}

void eqlin_oracle_backward_dx_group(int64_t G, const int64_t *mul, const int64_t *inv,
                                    int64_t Cp, int64_t Dp,
                                    const double *gy, const double *W,
                                    const int64_t *rows, int64_t n_out, double *dx)
{
    int64_t i;
#pragma omp parallel for schedule(dynamic, 1)
    for (i = 0; i < n_out; ++i) {
        const int64_t n = rows ? rows[i] : i;
        for (int64_t c = 0; c < Cp; ++c) {
            for (int64_t h = 0; h < G; ++h) {
                double acc = 0.0;
                for (int64_t d = 0; d < Dp; ++d)
                    for (int64_t g = 0; g < G; ++g)
                        acc += W[(d * Cp + c) * G + mul[inv[h] * G + g]] *
                               gy[n * Dp * G + d * G + g];
                dx[i * Cp * G + c * G + h] = acc;
            }
        }
    }
}

void eqlin_oracle_backward_dw_group(int64_t G, const int64_t *mul, int64_t Cp, int64_t Dp, int64_t N,
                                    const double *x, const double *gy, double *dW, double *db)
{
    int64_t j;
#pragma omp parallel for schedule(dynamic, 1)
    for (j = 0; j < Dp * Cp; ++j) {
        const int64_t d = j / Cp, c = j % Cp;
        for (int64_t u = 0; u < G; ++u) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
                for (int64_t h = 0; h < G; ++h)
                    acc += x[n * Cp * G + c * G + h] * gy[n * Dp * G + d * G + mul[h * G + u]];
            dW[j * G + u] = acc;
        }
    }
    if (db) {
        int64_t d;
#pragma omp parallel for schedule(static)
        for (d = 0; d < Dp; ++d) {
            double acc = 0.0;
            for (int64_t n = 0; n < N; ++n)
                for (int64_t g = 0; g < G; ++g)
                    acc += gy[n * Dp * G + d * G + g];
            db[d] = acc;
        }
    }
}

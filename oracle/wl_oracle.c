/*
 * Oracle for the theta-bundle linear.  TEST INFRASTRUCTURE ONLY: it is called
 * by the tests, by the smoke check and by the bench's CPU-baseline leg, never
 * by the product path.  It shares no code, header or helper with the CUDA
 * library.
 *
 * What it computes ("Add a new model architecture", introduction: a theta
 * bundle rebuilds one projection's weight as y = s.(W0 x) + U.(V^T x)):
 *
 *     y[m][n] = s[n] * sum_k W0[n][k] x[m][k]  +  sum_j U[n][j] T[m][j],
 *     T[m][j] = sum_k V[k][j] x[m][k]
 *
 * Layouts: x M x K, W0 N x K, U N x r, V K x r, y M x N, all row-major.
 * bf16 operands arrive as raw 16-bit patterns and are widened exactly
 * (bf16 -> fp32 -> fp64); s is fp32 widened to fp64.  Every sum runs in fp64,
 * single-threaded, in ascending index order, with no blocking or reordering.
 *
 * A second, independent path (wl_oracle_forward_dense) builds the effective
 * weight W_eff = diag(s) W0 + U V^T densely (the "precompute-outside" form on
 * the same page, "Override the graph build", step 5) and applies it to x.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

static double widen_bf16(uint16_t bits)
{
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* Factored form.  Returns 0 on success, -1 on allocation failure. */
int wl_oracle_forward(const uint16_t *x, const uint16_t *W0, const float *s,
                      const uint16_t *U, const uint16_t *V, double *y,
                      long M, long N, long K, long r)
{
    double *T = NULL;
    if (r > 0) {
        T = (double *)malloc(sizeof(double) * (size_t)(M * r));
        if (!T)
            return -1;
        /* T = V^T x, one column of x at a time */
        for (long m = 0; m < M; ++m)
            for (long j = 0; j < r; ++j) {
                double acc = 0.0;
                for (long k = 0; k < K; ++k)
                    acc += widen_bf16(V[k * r + j]) * widen_bf16(x[m * K + k]);
                T[m * r + j] = acc;
            }
    }
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n) {
            double z = 0.0; /* (W0 x)[n] */
            for (long k = 0; k < K; ++k)
                z += widen_bf16(W0[n * K + k]) * widen_bf16(x[m * K + k]);
            double d = 0.0; /* (U T)[n] */
            for (long j = 0; j < r; ++j)
                d += widen_bf16(U[n * r + j]) * T[m * r + j];
            y[m * N + n] = (double)s[n] * z + d;
        }
    free(T);
    return 0;
}

/* Dense form: W_eff = diag(s) W0 + U V^T, then y = W_eff x.  Small cases only
 * (it holds N*K doubles). */
int wl_oracle_forward_dense(const uint16_t *x, const uint16_t *W0, const float *s,
                            const uint16_t *U, const uint16_t *V, double *y,
                            long M, long N, long K, long r)
{
    double *Weff = (double *)malloc(sizeof(double) * (size_t)(N * K));
    if (!Weff)
        return -1;
    for (long n = 0; n < N; ++n)
        for (long k = 0; k < K; ++k) {
            double uv = 0.0;
            for (long j = 0; j < r; ++j)
                uv += widen_bf16(U[n * r + j]) * widen_bf16(V[k * r + j]);
            Weff[n * K + k] = (double)s[n] * widen_bf16(W0[n * K + k]) + uv;
        }
    for (long m = 0; m < M; ++m)
        for (long n = 0; n < N; ++n) {
            double acc = 0.0;
            for (long k = 0; k < K; ++k)
                acc += Weff[n * K + k] * widen_bf16(x[m * K + k]);
            y[m * N + n] = acc;
        }
    free(Weff);
    return 0;
}

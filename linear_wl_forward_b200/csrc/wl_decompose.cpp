// Host-side decomposition of dense layer weights into theta bundles:
//   band mean W0, least-squares per-row scale s, truncated SVD of the residual.
// ("Quality", "Why sharing fails: reconstruction error": the band-mean W0,
// the per-layer residual weight - s.W0 and its rank-r delta; "Add a new model
// architecture", "Decompose HF weights", step 4.)
//
// The SVD is a one-sided Jacobi (Hestenes) iteration in fp64 over the columns
// of the residual or of its transpose, whichever has fewer columns: pairs of
// columns are rotated until all pairs are orthogonal; the column norms are then
// the singular values and the accumulated rotation gives the other side.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <new>
#include <numeric>
#include <vector>

#include "../../include/wl.h"

namespace {

constexpr int kJacobiMaxSweeps = 80;

// A is m x n column-major (n <= m).  On return its columns are mutually
// orthogonal (A_in Q) and Q (n x n, column-major) holds the rotations.  A pair
// counts as orthogonal once |<a_i, a_j>| <= tol ||a_i|| ||a_j||, tol = m times
// the fp64 unit roundoff (the rounding level of the length-m dot product
// itself; a tighter test can keep rotating on rounding noise).  Returns false
// if a sweep still rotated after kJacobiMaxSweeps sweeps.
bool jacobi_orthogonalize(std::vector<double> &A, int m, int n, std::vector<double> &Q) {
    Q.assign((size_t)n * n, 0.0);
    for (int i = 0; i < n; ++i) Q[(size_t)i * n + i] = 1.0;
    const double eps = std::max(1e-15, (double)m * 1.1102230246251565e-16);
    for (int sweep = 0; sweep < kJacobiMaxSweeps; ++sweep) {
        bool rotated = false;
        for (int i = 0; i < n - 1; ++i) {
            double *ai = &A[(size_t)i * m];
            for (int j = i + 1; j < n; ++j) {
                double *aj = &A[(size_t)j * m];
                double alpha = 0, beta = 0, gamma = 0;
                for (int k = 0; k < m; ++k) {
                    alpha += ai[k] * ai[k];
                    beta += aj[k] * aj[k];
                    gamma += ai[k] * aj[k];
                }
                if (gamma == 0.0 || std::fabs(gamma) <= eps * std::sqrt(alpha * beta)) continue;
                rotated = true;
                const double zeta = (beta - alpha) / (2.0 * gamma);
                const double t = (zeta >= 0 ? 1.0 : -1.0) / (std::fabs(zeta) + std::sqrt(1.0 + zeta * zeta));
                const double c = 1.0 / std::sqrt(1.0 + t * t);
                const double s = c * t;
                for (int k = 0; k < m; ++k) {
                    const double x = ai[k], y = aj[k];
                    ai[k] = c * x - s * y;
                    aj[k] = s * x + c * y;
                }
                double *qi = &Q[(size_t)i * n], *qj = &Q[(size_t)j * n];
                for (int k = 0; k < n; ++k) {
                    const double x = qi[k], y = qj[k];
                    qi[k] = c * x - s * y;
                    qj[k] = s * x + c * y;
                }
            }
        }
        if (!rotated) return true;
    }
    return false;
}

// Rank-r truncated SVD of R (N x K, row-major): U = P_r S_r (N x r), V = Q_r (K x r).
// Returns false if the Jacobi iteration did not converge (the factors are
// then those of the last sweep).
bool truncated_svd(const std::vector<double> &R, int N, int K, int r, double *U, double *V) {
    std::fill(U, U + (size_t)N * r, 0.0);
    std::fill(V, V + (size_t)K * r, 0.0);
    if (r == 0) return true;
    const bool cols_are_k = K <= N;  // orthogonalise the K columns of R, else the N columns of R^T
    const int m = cols_are_k ? N : K, n = cols_are_k ? K : N;
    std::vector<double> A((size_t)m * n);
    for (int a = 0; a < N; ++a)
        for (int b = 0; b < K; ++b) {
            if (cols_are_k)
                A[(size_t)b * m + a] = R[(size_t)a * K + b];  // column b of R
            else
                A[(size_t)a * m + b] = R[(size_t)a * K + b];  // column a of R^T
        }
    std::vector<double> Q;
    const bool converged = jacobi_orthogonalize(A, m, n, Q);
    std::vector<double> sigma(n);
    for (int i = 0; i < n; ++i) {
        double ss = 0;
        for (int k = 0; k < m; ++k) ss += A[(size_t)i * m + k] * A[(size_t)i * m + k];
        sigma[i] = std::sqrt(ss);
    }
    std::vector<int> order(n);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return sigma[a] > sigma[b]; });
    const int kk = std::min(r, n);
    for (int c = 0; c < kk; ++c) {
        const int i = order[c];
        const double sg = sigma[i];
        if (sg == 0.0) continue;  // zero singular value: leave the column zero
        const double *col = &A[(size_t)i * m];
        const double *q = &Q[(size_t)i * n];
        if (cols_are_k) {
            // R Q = A: column i of A is sigma_i p_i (length N); Q column is v_i (length K)
            for (int a = 0; a < N; ++a) U[(size_t)a * r + c] = col[a];
            for (int b = 0; b < K; ++b) V[(size_t)b * r + c] = q[b];
        } else {
            // R^T Q = A: R = Q A^T; left vectors are Q columns (length N), right A/sigma (length K)
            for (int a = 0; a < N; ++a) U[(size_t)a * r + c] = q[a] * sg;
            for (int b = 0; b < K; ++b) V[(size_t)b * r + c] = col[b] / sg;
        }
    }
    return converged;
}

double rel_err_fp64(const float *W, const float *W0, const float *s, const float *U, const float *V,
                    int N, int K, int r) {
    double num = 0, den = 0;
    for (int n = 0; n < N; ++n)
        for (int k = 0; k < K; ++k) {
            double uv = 0;
            for (int j = 0; j < r; ++j) uv += (double)U[(size_t)n * r + j] * (double)V[(size_t)k * r + j];
            const double w = W[(size_t)n * K + k];
            const double d = w - ((double)s[n] * (double)W0[(size_t)n * K + k] + uv);
            num += d * d;
            den += w * w;
        }
    return den > 0 ? std::sqrt(num / den) : std::sqrt(num);
}

// Row n of U_l V_l^T (fp64 factors) into out[K].
void uv_row(const double *Ul, const double *Vl, int n, int K, int r, double *out) {
    for (int k = 0; k < K; ++k) {
        double acc = 0;
        for (int j = 0; j < r; ++j) acc += Ul[(size_t)n * r + j] * Vl[(size_t)k * r + j];
        out[k] = acc;
    }
}

// Band-mean start, then `iters` alternating least-squares iterations ("Quality
// (Gemma 4 31B)", "ALS optimization barely helps"), each of three exact
// block updates of the total squared residual: every band's W0 with s and
// U V^T fixed, every s with W0 and U V^T fixed, every U V^T (truncated SVD of
// W_l - diag(s_l) W0) with W0 and s fixed.
wl_status decompose_impl(const float *W, int L, int N, int K, int G, int r, const int *band_of_layer, int iters,
                         float *W0, float *s, float *U, float *V, double *rel_err) {
    if (!W || !W0 || !s || (r > 0 && (!U || !V))) return WL_ERR_INVALID_ARG;
    if (L < 1 || N < 1 || K < 1 || G < 1 || r < 0 || iters < 0) return WL_ERR_INVALID_ARG;
    try {
        std::vector<int> band(L);
        for (int l = 0; l < L; ++l) {
            band[l] = band_of_layer ? band_of_layer[l] : (int)(((long long)l * G) / L);
            if (band[l] < 0 || band[l] >= G) return WL_ERR_INVALID_ARG;
        }
        const size_t NK = (size_t)N * K;
        std::vector<double> w0((size_t)G * NK, 0.0);
        std::vector<int> count(G, 0);
        for (int l = 0; l < L; ++l) {
            ++count[band[l]];
            double *dst = &w0[(size_t)band[l] * NK];
            const float *src = W + (size_t)l * NK;
            for (size_t i = 0; i < NK; ++i) dst[i] += src[i];
        }
        for (int b = 0; b < G; ++b)
            if (count[b] > 0)
                for (size_t i = 0; i < NK; ++i) w0[(size_t)b * NK + i] /= count[b];
        std::vector<double> sd((size_t)L * N, 1.0);
        std::vector<double> Ud((size_t)L * N * r, 0.0), Vd((size_t)L * K * r, 0.0);
        std::vector<double> R(NK), uv(K);
        // s_l[n] = <W_l[n] - (U_l V_l^T)[n], W0_b[n]> / ||W0_b[n]||^2 (1 for a zero row)
        auto fit_scales = [&](int l, bool with_uv) {
            const float *w = W + (size_t)l * NK;
            const double *b0 = &w0[(size_t)band[l] * NK];
            for (int n = 0; n < N; ++n) {
                if (with_uv && r > 0) uv_row(&Ud[(size_t)l * N * r], &Vd[(size_t)l * K * r], n, K, r, uv.data());
                double num = 0, den = 0;
                for (int k = 0; k < K; ++k) {
                    const double t = (double)w[(size_t)n * K + k] - (with_uv && r > 0 ? uv[k] : 0.0);
                    num += t * b0[(size_t)n * K + k];
                    den += b0[(size_t)n * K + k] * b0[(size_t)n * K + k];
                }
                sd[(size_t)l * N + n] = den > 0 ? num / den : 1.0;
            }
        };
        // U_l V_l^T = rank-r truncated SVD of W_l - diag(s_l) W0_b
        bool converged = true;
        auto fit_delta = [&](int l) {
            if (r == 0) return;
            const float *w = W + (size_t)l * NK;
            const double *b0 = &w0[(size_t)band[l] * NK];
            for (int n = 0; n < N; ++n)
                for (int k = 0; k < K; ++k)
                    R[(size_t)n * K + k] = (double)w[(size_t)n * K + k] - sd[(size_t)l * N + n] * b0[(size_t)n * K + k];
            if (!truncated_svd(R, N, K, r, &Ud[(size_t)l * N * r], &Vd[(size_t)l * K * r])) converged = false;
        };
        for (int l = 0; l < L; ++l) {
            fit_scales(l, false);
            fit_delta(l);
        }
        std::vector<double> num(K);
        for (int it = 0; it < iters; ++it) {
            // W0_b[n] = sum_l s_l[n] (W_l[n] - (U_l V_l^T)[n]) / sum_l s_l[n]^2 (kept if all s are 0)
            for (int b = 0; b < G; ++b) {
                for (int n = 0; n < N; ++n) {
                    std::fill(num.begin(), num.end(), 0.0);
                    double den = 0;
                    for (int l = 0; l < L; ++l) {
                        if (band[l] != b) continue;
                        const double sc = sd[(size_t)l * N + n];
                        const float *w = W + (size_t)l * NK + (size_t)n * K;
                        if (r > 0) uv_row(&Ud[(size_t)l * N * r], &Vd[(size_t)l * K * r], n, K, r, uv.data());
                        for (int k = 0; k < K; ++k) num[k] += sc * ((double)w[k] - (r > 0 ? uv[k] : 0.0));
                        den += sc * sc;
                    }
                    if (den > 0)
                        for (int k = 0; k < K; ++k) w0[(size_t)b * NK + (size_t)n * K + k] = num[k] / den;
                }
            }
            for (int l = 0; l < L; ++l) fit_scales(l, true);
            for (int l = 0; l < L; ++l) fit_delta(l);
        }
        for (size_t i = 0; i < (size_t)G * NK; ++i) W0[i] = (float)w0[i];
        for (size_t i = 0; i < (size_t)L * N; ++i) s[i] = (float)sd[i];
        if (r > 0) {
            for (size_t i = 0; i < Ud.size(); ++i) U[i] = (float)Ud[i];
            for (size_t i = 0; i < Vd.size(); ++i) V[i] = (float)Vd[i];
        }
        if (rel_err)
            for (int l = 0; l < L; ++l)
                rel_err[l] = rel_err_fp64(W + (size_t)l * NK, W0 + (size_t)band[l] * NK, s + (size_t)l * N,
                                          r > 0 ? U + (size_t)l * N * r : nullptr,
                                          r > 0 ? V + (size_t)l * K * r : nullptr, N, K, r);
        if (!converged) return WL_ERR_NOT_CONVERGED;
    } catch (const std::bad_alloc &) {
        return WL_ERR_NOMEM;
    }
    return WL_OK;
}

}  // namespace

extern "C" {

wl_status wl_decompose(const float *W, int L, int N, int K, int G, int r, const int *band_of_layer,
                       float *W0, float *s, float *U, float *V, double *rel_err) {
    return decompose_impl(W, L, N, K, G, r, band_of_layer, 0, W0, s, U, V, rel_err);
}

wl_status wl_decompose_als(const float *W, int L, int N, int K, int G, int r, const int *band_of_layer,
                           int iters, float *W0, float *s, float *U, float *V, double *rel_err) {
    return decompose_impl(W, L, N, K, G, r, band_of_layer, iters, W0, s, U, V, rel_err);
}

double wl_relative_frobenius_error(const float *W, const float *W0, const float *s, const float *U,
                                   const float *V, int N, int K, int r) {
    if (!W || !W0 || !s || N < 1 || K < 1 || r < 0 || (r > 0 && (!U || !V))) return -1.0;
    return rel_err_fp64(W, W0, s, U, V, N, K, r);
}

}  // extern "C"

"""Pins for the decomposition oracle (CPU only): the pages' passthrough result,
closed forms and invariants that hold for any weights."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))


def rand_w(seed, L, N, K):
    return np.random.default_rng(seed).standard_normal((L, N, K))


@pytest.mark.parametrize("r", GOLDEN["passthrough_error"]["ranks"])
def test_passthrough_is_exact_for_every_rank(r):
    """G = number of layers: W0 = W, s = 1 exactly, residual 0, error 0
    (pages: error exactly zero at G = 26 for ranks 4-256)."""
    L, N, K = 3, 10, 14
    W = rand_w(1, L, N, K)
    W0, s, U, V = oracle.decompose(W, G=L, r=r)
    for l in range(L):
        assert np.array_equal(W0[l], W[l])
        assert np.array_equal(s[l], np.ones(N))
        assert np.max(np.abs(U[l] @ V[l].T)) == 0.0
        e = oracle.relative_frobenius_error(W[l], W0[l], s[l], U[l], V[l])
        assert e == GOLDEN["passthrough_error"]["value"]


def test_band_mean_and_scalar_multiples():
    """Layers W_l = c_l A in one band: W0 = mean(c) A, s_l = c_l / mean(c),
    zero residual (closed form of the band mean and least-squares scale)."""
    rng = np.random.default_rng(2)
    A = rng.standard_normal((8, 12))
    c = np.array([0.5, 1.5, 2.0, -1.0])
    W = c[:, None, None] * A[None]
    W0, s, U, V = oracle.decompose(W, G=1, r=2)
    cbar = c.mean()
    assert np.allclose(W0[0], cbar * A, atol=1e-14)
    for l in range(4):
        assert np.allclose(s[l], c[l] / cbar, atol=1e-13)
        assert oracle.relative_frobenius_error(W[l], W0[0], s[l], U[l], V[l]) < 1e-12


def test_least_squares_residual_orthogonal_to_w0_rows():
    W = rand_w(3, 4, 9, 11)
    W0, s, U, V = oracle.decompose(W, G=2, r=0)
    bands = oracle.band_of_layer_contiguous(4, 2)
    for l in range(4):
        R = W[l] - s[l][:, None] * W0[bands[l]]
        dots = np.einsum("nk,nk->n", R, W0[bands[l]])
        assert np.max(np.abs(dots)) < 1e-12


def test_error_non_increasing_in_rank_and_eckart_young():
    """e(r) falls with r, and ||W||^2 e(r)^2 equals the tail energy of the
    residual spectrum (eigenvalues of R R^T, computed by a different routine)."""
    L, N, K = 4, 10, 16
    W = rand_w(4, L, N, K)
    bands = oracle.band_of_layer_contiguous(L, 1)
    prev = np.inf
    for r in range(0, 11):
        W0, s, U, V = oracle.decompose(W, G=1, r=r)
        e = oracle.relative_frobenius_error(W[1], W0[0], s[1], U[1], V[1])
        assert e <= prev + 1e-15
        prev = e
        R = W[1] - s[1][:, None] * W0[bands[1]]
        lam = np.sort(np.linalg.eigvalsh(R @ R.T))[::-1]
        tail = max(float(np.sum(lam[r:])), 0.0)
        assert abs(np.linalg.norm(W[1]) ** 2 * e ** 2 - tail) < 1e-9 * np.linalg.norm(W[1]) ** 2
    assert prev < 1e-12  # r >= rank(R) reconstructs exactly


def test_factors_orthonormal_and_sigma_in_u():
    W = rand_w(5, 3, 12, 9)
    W0, s, U, V = oracle.decompose(W, G=1, r=5)
    for l in range(3):
        assert np.allclose(V[l].T @ V[l], np.eye(5), atol=1e-12)
        G = U[l].T @ U[l]
        assert np.allclose(G, np.diag(np.diag(G)), atol=1e-10)  # U columns orthogonal
        assert np.all(np.diff(np.diag(G)) <= 1e-12)               # sigma descending


def test_rank_beyond_matrix_is_zero_padded():
    W = rand_w(6, 2, 5, 4)
    W0, s, U, V = oracle.decompose(W, G=1, r=9)
    assert U.shape == (2, 5, 9) and V.shape == (2, 4, 9)
    assert np.all(U[:, :, 4:] == 0) and np.all(V[:, :, 4:] == 0)


def test_explicit_interleaved_bands():
    W = rand_w(7, 4, 6, 5)
    W0, s, U, V = oracle.decompose(W, G=2, r=1, band_of_layer=[0, 1, 0, 1])
    assert np.allclose(W0[0], (W[0] + W[2]) / 2)
    assert np.allclose(W0[1], (W[1] + W[3]) / 2)


# ------------------------------------------------------------- ALS refinement --
@pytest.mark.parametrize("G,r,bands", [(1, 0, None), (1, 3, None), (2, 2, None), (2, 1, [0, 1, 1, 0])])
def test_als_objective_never_increases(G, r, bands):
    """Every ALS step is an exact least-squares minimisation over its block of
    unknowns, so the total squared residual cannot grow at any step."""
    W = rand_w(20 + G + r, 4, 7, 9)
    trace = []
    oracle.decompose_als(W, G, r, iters=6, band_of_layer=bands, trace=trace)
    for a, b in zip(trace, trace[1:]):
        assert b <= a * (1 + 1e-12) + 1e-12


def test_als_zero_iterations_is_the_mean_start():
    W = rand_w(21, 3, 6, 5)
    a = oracle.decompose(W, G=1, r=2)
    b = oracle.decompose_als(W, G=1, r=2, iters=0)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_als_rank0_converges_to_best_rank1_per_row():
    """With r = 0 and one band the objective separates over rows: row n of all
    layers is an L x K matrix M_n fitted by s[:, n] W0[n]^T, a rank-1 model,
    and ALS is an alternating power iteration.  It must reach the Eckart-Young
    optimum sum_n sum_{i >= 2} sigma_i(M_n)^2 (numpy's SVD of each M_n)."""
    W = rand_w(22, 4, 5, 6)
    trace = []
    oracle.decompose_als(W, G=1, r=0, iters=300, trace=trace)
    best = sum(float(np.sum(np.linalg.svd(W[:, n, :], compute_uv=False)[1:] ** 2)) for n in range(W.shape[1]))
    assert abs(trace[-1] - best) <= 1e-9 * best
    assert trace[0] > best * (1 + 1e-3)  # the mean start is not already optimal


def test_als_hand_example_two_layers():
    """W_1 = [2, 0], W_2 = [0, 1] (one row, one band, r = 0): the stacked 2 x 2
    matrix has singular values 2 and 1, so ALS must approach a residual of
    1^2 = 1 with W0 along [1, 0] and the second layer's scale -> 0; the mean
    start (W0 = [1, 0.5]) has residual 1.6."""
    W = np.array([[[2.0, 0.0]], [[0.0, 1.0]]])
    trace = []
    W0, s, U, V = oracle.decompose_als(W, G=1, r=0, iters=60, trace=trace)
    assert trace[0] == pytest.approx(1.6, abs=1e-12)
    assert trace[-1] == pytest.approx(1.0, abs=1e-12)
    assert abs(W0[0, 0, 1]) <= 1e-12 * abs(W0[0, 0, 0])
    assert abs(s[1, 0]) <= 1e-12


def test_als_keeps_passthrough_exact():
    W = rand_w(23, 3, 5, 7)
    W0, s, U, V = oracle.decompose_als(W, G=3, r=2, iters=3)
    for l in range(3):
        assert oracle.relative_frobenius_error(W[l], W0[l], s[l], U[l], V[l]) <= 1e-15

"""The library's host decomposition (wl_decompose, one-sided Jacobi SVD in C++)
against the numpy oracle (CPU only).  SVD factors are not unique (signs,
rotations inside repeated singular values), so the comparison is on W0, s, the
product U V^T and the errors."""
import numpy as np
import pytest

import linear_wl_forward_b200 as wl
import oracle
from linear_wl_forward_b200 import build as wlbuild


@pytest.fixture(scope="module", autouse=True)
def _built():
    wlbuild.build()


@pytest.mark.parametrize("L,N,K,G,r", [(4, 12, 20, 2, 3), (3, 24, 10, 1, 5), (2, 9, 9, 2, 4),
                                       (6, 16, 16, 3, 16), (5, 7, 30, 1, 0)])
def test_matches_oracle(L, N, K, G, r):
    W = np.random.default_rng(L * 100 + N + K).standard_normal((L, N, K)).astype(np.float32)
    W0, s, U, V, err = wl.decompose(W, G, r)
    oW0, os_, oU, oV = oracle.decompose(W.astype(np.float64), G, r)
    bands = oracle.band_of_layer_contiguous(L, G)
    assert np.allclose(W0, oW0, atol=1e-6)
    assert np.allclose(s, os_, atol=1e-5)
    for l in range(L):
        uv = U[l].astype(np.float64) @ V[l].astype(np.float64).T
        ouv = oU[l] @ oV[l].T
        assert np.max(np.abs(uv - ouv)) <= 1e-4 * max(1.0, np.max(np.abs(ouv)))
        oe = oracle.relative_frobenius_error(W[l], oW0[bands[l]], os_[l], oU[l], oV[l])
        assert abs(err[l] - oe) < 1e-5
        e2 = wl.relative_frobenius_error(W[l], W0[bands[l]], s[l], U[l] if r else None,
                                         V[l] if r else None)
        assert abs(e2 - err[l]) < 1e-12


def test_passthrough_zero_error():
    W = np.random.default_rng(3).standard_normal((3, 10, 12)).astype(np.float32)
    W0, s, U, V, err = wl.decompose(W, 3, 4)
    assert np.array_equal(W0, W)
    assert np.all(s == 1.0)
    assert np.all(err == 0.0)


def test_interleaved_bands_and_errors():
    W = np.random.default_rng(4).standard_normal((4, 8, 6)).astype(np.float32)
    W0, s, U, V, err = wl.decompose(W, 2, 2, band_of_layer=[1, 0, 1, 0])
    assert np.allclose(W0[1], (W[0] + W[2]) / 2, atol=1e-6)
    with pytest.raises(wl.WLError):
        wl.decompose(W, 2, 2, band_of_layer=[0, 1, 2, 0])


def test_error_non_increasing_in_rank():
    W = np.random.default_rng(5).standard_normal((3, 12, 18)).astype(np.float32)
    prev = np.inf
    for r in range(0, 13, 2):
        err = wl.decompose(W, 1, r)[4]
        assert err.mean() <= prev + 1e-6
        prev = err.mean()
    assert prev < 1e-5


@pytest.mark.parametrize("L,N,K,G,r,iters,bands", [(4, 12, 20, 2, 3, 3, None), (3, 9, 14, 1, 0, 5, None),
                                                   (4, 10, 8, 2, 2, 2, [0, 1, 1, 0]), (2, 6, 6, 1, 4, 4, None)])
def test_als_matches_oracle(L, N, K, G, r, iters, bands):
    """wl_decompose_als against the numpy ALS oracle: W0, s, U V^T and the
    errors after the same number of rounds."""
    W = np.random.default_rng(L * 1000 + N * 10 + K + iters).standard_normal((L, N, K)).astype(np.float32)
    W0, s, U, V, err = wl.decompose(W, G, r, band_of_layer=bands, als_iters=iters)
    oW0, os_, oU, oV = oracle.decompose_als(W.astype(np.float64), G, r, iters, band_of_layer=bands)
    b = oracle.band_of_layer_contiguous(L, G) if bands is None else bands
    assert np.allclose(W0, oW0, atol=1e-5, rtol=1e-5)
    assert np.allclose(s, os_, atol=1e-5, rtol=1e-5)
    for l in range(L):
        uv = U[l].astype(np.float64) @ V[l].astype(np.float64).T
        ouv = oU[l] @ oV[l].T
        assert np.max(np.abs(uv - ouv)) <= 1e-4 * max(1.0, np.max(np.abs(ouv)))
        oe = oracle.relative_frobenius_error(W[l], oW0[b[l]], os_[l], oU[l], oV[l])
        assert abs(err[l] - oe) < 1e-5


def test_als_zero_rounds_is_plain_decompose_and_rounds_do_not_hurt():
    W = np.random.default_rng(9).standard_normal((4, 10, 12)).astype(np.float32)
    a = wl.decompose(W, 1, 2)
    b = wl.decompose(W, 1, 2, als_iters=0)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    c = wl.decompose(W, 1, 2, als_iters=4)
    # the total squared residual can only go down; per layer it may move either way
    total = lambda e: float(np.sum(e ** 2 * np.sum(W.astype(np.float64) ** 2, axis=(1, 2))))
    assert total(c[4]) <= total(a[4]) * (1 + 1e-6)


def test_als_rejects_negative_rounds():
    W = np.zeros((2, 3, 4), np.float32)
    with pytest.raises(wl.WLError):
        wl.decompose(W, 1, 1, als_iters=-1)


def test_gemma3_shape_matches_oracle_and_converges():
    """One Gemma-3-1B-shaped family at a size the host SVD meets in practice
    (two layers of 256 x 1152, one band, rank 16): the Jacobi iteration
    converges (no WL_ERR_NOT_CONVERGED) and the bundle matches the numpy
    oracle's (W0, s, U V^T and the errors)."""
    import time

    rng = np.random.default_rng(11)
    W = (0.02 * rng.standard_normal((2, 256, 1152))).astype(np.float32)
    t0 = time.perf_counter()
    W0, s, U, V, err = wl.decompose(W, 1, 16)
    assert time.perf_counter() - t0 < 120
    oW0, os_, oU, oV = oracle.decompose(W.astype(np.float64), 1, 16)
    assert np.allclose(W0, oW0, atol=1e-7)
    assert np.allclose(s, os_, atol=1e-5)
    for l in range(2):
        uv = U[l].astype(np.float64) @ V[l].astype(np.float64).T
        ouv = oU[l] @ oV[l].T
        assert np.max(np.abs(uv - ouv)) <= 1e-4 * np.max(np.abs(ouv))
        oe = oracle.relative_frobenius_error(W[l], oW0[0], os_[l], oU[l], oV[l])
        assert abs(err[l] - oe) < 1e-5

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

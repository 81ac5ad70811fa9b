"""Pins for the forward oracle (CPU only).

Each test pins the oracle to something other than itself: a hand-derived tiny
case, exact integer arithmetic, the dense effective-weight definition, a
textbook matmul special case, and algebraic invariants.  Together they fail on
a dropped term (s or U.T), a sign error, a wrong index or a transposed operand.
"""
import itertools

import numpy as np
import pytest
import torch

import oracle
import wl_inputs


def bf(vals):
    return torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16)


def test_hand_computed_2x2_rank1():
    # W0 = [[1,2],[3,4]], s = [2, 0.5], U = [[1],[-1]], V = [[1],[1]], x = [1, 1]
    # W0 x = [3, 7]; V^T x = 2; y = [2*3 + 1*2, 0.5*7 - 1*2] = [8, 1.5]
    y = oracle.forward(bf([[1, 1]]), bf([[1, 2], [3, 4]]),
                       torch.tensor([2.0, 0.5]), bf([[1], [-1]]), bf([[1], [1]]))
    assert y.tolist() == [[8.0, 1.5]]


def test_hand_computed_rank2_asymmetric():
    # N=3, K=2, r=2; chosen so that swapping U<->V roles or transposing fails.
    # W0 x = [1*2+0*3, 0*2+1*3, 1*2+1*3] = [2, 3, 5]
    # V = [[1, 0], [2, -1]] (K x r): T = V^T x = [1*2+2*3, 0*2-1*3] = [8, -3]
    # U = [[1, 0], [0, 1], [1, 1]] (N x r): U T = [8, -3, 5]
    # s = [1, 2, -1]: y = [2+8, 6-3, -5+5] = [10, 3, 0]
    y = oracle.forward(bf([[2, 3]]), bf([[1, 0], [0, 1], [1, 1]]),
                       torch.tensor([1.0, 2.0, -1.0]),
                       bf([[1, 0], [0, 1], [1, 1]]), bf([[1, 0], [2, -1]]))
    assert y.tolist() == [[10.0, 3.0, 0.0]]


def _int_case(rng, M, N, K, r):
    x = rng.integers(-3, 4, (M, K))
    W0 = rng.integers(-4, 5, (N, K))
    s = rng.integers(-2, 3, (N,)).astype(np.float64) * 0.5
    U = rng.integers(-3, 4, (N, r))
    V = rng.integers(-3, 4, (K, r))
    return x, W0, s, U, V


@pytest.mark.parametrize("M,N,K,r", [(1, 5, 7, 3), (3, 4, 9, 1), (2, 6, 3, 4), (2, 3, 4, 0)])
def test_exact_small_integers_bruteforce(M, N, K, r):
    """Small integers are exact in bf16 and in fp64: the oracle must equal
    pure-Python integer brute force bit for bit."""
    rng = np.random.default_rng(1000 + M * 100 + N * 10 + K + r)
    x, W0, s, U, V = _int_case(rng, M, N, K, r)
    want = [[0.0] * N for _ in range(M)]
    for m, n in itertools.product(range(M), range(N)):
        z = sum(int(W0[n, k]) * int(x[m, k]) for k in range(K))
        d = 0
        for j in range(r):
            t = sum(int(V[k, j]) * int(x[m, k]) for k in range(K))
            d += int(U[n, j]) * t
        want[m][n] = float(s[n]) * z + d
    got = oracle.forward(bf(x.tolist()), bf(W0.tolist()), torch.tensor(s, dtype=torch.float32),
                         bf(U.reshape(N, r).tolist()) if r else torch.zeros(N, 0, dtype=torch.bfloat16),
                         bf(V.reshape(K, r).tolist()) if r else torch.zeros(K, 0, dtype=torch.bfloat16))
    assert got.tolist() == want


@pytest.mark.parametrize("M,N,K,r", [(3, 37, 24, 5), (1, 8, 64, 16), (5, 19, 13, 7)])
def test_factored_equals_dense_effective_weight(M, N, K, r):
    """(diag(s) W0 + U V^T) x built densely equals the factored form."""
    c = wl_inputs.random_case(7 + M + N, M, N, K, r)
    p = c.projs[0]
    y = oracle.forward(c.x, p.W0, p.s, p.U, p.V)
    yd = oracle.forward_dense(c.x, p.W0, p.s, p.U, p.V)
    assert np.max(np.abs(y - yd)) <= 1e-12 * np.max(np.abs(yd))


def test_no_delta_unit_scale_is_plain_matmul():
    """U = 0 (r = 0) and s = 1 reduce the method to y = x W0^T."""
    c = wl_inputs.random_case(3, 4, 33, 40, 0)
    p = c.projs[0]
    ones = torch.ones(p.N)
    y = oracle.forward(c.x, p.W0, ones, p.U, p.V)
    ref = np.matmul(c.x.double().numpy(), p.W0.double().numpy().T)
    assert np.max(np.abs(y - ref)) <= 1e-13 * np.max(np.abs(ref))


def test_scale_only_applies_to_shared_block():
    """s multiplies W0 x only: with W0 = 0 the output is U V^T x for any s."""
    c = wl_inputs.random_case(4, 2, 16, 24, 3)
    p = c.projs[0]
    zero = torch.zeros_like(p.W0)
    y1 = oracle.forward(c.x, zero, p.s, p.U, p.V)
    y2 = oracle.forward(c.x, zero, torch.full_like(p.s, 7.0), p.U, p.V)
    ref = c.x.double().numpy() @ p.V.double().numpy() @ p.U.double().numpy().T
    assert np.allclose(y1, ref, rtol=0, atol=1e-14)
    assert np.allclose(y2, ref, rtol=0, atol=1e-14)


def test_linearity_and_rank_permutation():
    c = wl_inputs.random_case(5, 3, 21, 32, 6)
    p = c.projs[0]
    y = oracle.forward(c.x, p.W0, p.s, p.U, p.V)
    # doubling x is exact in bf16 and scales every term exactly
    y2 = oracle.forward((c.x.float() * 2).to(torch.bfloat16), p.W0, p.s, p.U, p.V)
    assert np.array_equal(y2, 2 * y)
    # permuting the rank index of U and V together leaves U V^T unchanged
    perm = torch.tensor([3, 0, 5, 1, 4, 2])
    yp = oracle.forward(c.x, p.W0, p.s, p.U[:, perm], p.V[:, perm])
    assert np.max(np.abs(yp - y)) <= 1e-12 * np.max(np.abs(y))


def test_decomposed_passthrough_reproduces_dense_matmul():
    """G = L: W0 = W, s = 1, zero residual, so the forward equals W x."""
    rng = np.random.default_rng(11)
    L, N, K, r = 2, 12, 16, 4
    W = rng.standard_normal((L, N, K))
    W0, s, U, V = oracle.decompose(W, G=L, r=r)
    # round the (exact) passthrough bundle to bf16: W0 = W up to that rounding
    x = bf(rng.standard_normal((3, K)).tolist())
    for l in range(L):
        W0b = torch.tensor(W0[l]).to(torch.bfloat16)
        y = oracle.forward(x, W0b, torch.tensor(s[l], dtype=torch.float32),
                           torch.tensor(U[l]).to(torch.bfloat16), torch.tensor(V[l]).to(torch.bfloat16))
        ref = x.double().numpy() @ W0b.double().numpy().T
        assert np.max(np.abs(y - ref)) <= 1e-12

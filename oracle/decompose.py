"""Decomposition oracle (numpy, fp64).  TEST INFRASTRUCTURE ONLY.

Per projection family and band b with member layers L_b (pages: "Quality",
"Why sharing fails: reconstruction error"; "Add a new model architecture",
"Decompose HF weights"):

1. W0_b = mean of the band's per-layer weights ("the band-mean W0").
2. s_l[n] = <W_l[n,:], W0_b[n,:]> / ||W0_b[n,:]||^2 -- the per-row scale, read
   as the least-squares fit of each row of W_l onto the same row of W0_b (the
   pages name a "per-row scale" without a formula).  A zero W0 row gives s = 1.
3. R_l = W_l - diag(s_l) W0_b ("the per-layer residual weight - s.W0").
4. Truncated SVD R_l = P S Q^T; U_l = P[:, :r] S[:r], V_l = Q[:, :r] (the
   singular values go into U -- the split is not stated on the pages).  Widths
   beyond rank(R_l) are zero-padded.
5. relative Frobenius error ||W_l - (diag(s_l) W0_b + U_l V_l^T)||_F / ||W_l||_F.

``numpy.linalg.svd`` serves as the library SVD step.  ``decompose_als``
refines the mean start by alternating least squares (see there).
"""
from __future__ import annotations

import numpy as np


def band_of_layer_contiguous(L: int, G: int):
    """Contiguous equal bands: band(l) = floor(l * G / L)."""
    return [(l * G) // L for l in range(L)]


def decompose(W, G: int, r: int, band_of_layer=None):
    """W: (L, N, K) array.  Returns (W0 (G,N,K), s (L,N), U (L,N,r), V (L,K,r))
    in fp64."""
    W = np.asarray(W, dtype=np.float64)
    L, N, K = W.shape
    bands = band_of_layer_contiguous(L, G) if band_of_layer is None else list(band_of_layer)
    W0 = np.zeros((G, N, K))
    for b in range(G):
        members = [l for l in range(L) if bands[l] == b]
        if members:
            W0[b] = np.mean(W[members], axis=0)
    s = np.empty((L, N))
    U = np.zeros((L, N, r))
    V = np.zeros((L, K, r))
    for l in range(L):
        w0 = W0[bands[l]]
        num = np.einsum("nk,nk->n", W[l], w0)
        den = np.einsum("nk,nk->n", w0, w0)
        s[l] = np.where(den > 0, num / np.where(den > 0, den, 1.0), 1.0)
        R = W[l] - s[l][:, None] * w0
        if r > 0:
            P, sig, Qt = np.linalg.svd(R, full_matrices=False)
            kk = min(r, sig.shape[0])
            U[l, :, :kk] = P[:, :kk] * sig[:kk]
            V[l, :, :kk] = Qt[:kk].T
    return W0, s, U, V


def theta_reconstruct(W0b, s, U, V):
    """diag(s) W0 + U V^T for one layer."""
    return np.asarray(s)[:, None] * np.asarray(W0b) + np.asarray(U) @ np.asarray(V).T


def relative_frobenius_error(W, W0b, s, U, V) -> float:
    W = np.asarray(W, dtype=np.float64)
    R = W - theta_reconstruct(W0b, s, U, V)
    return float(np.linalg.norm(R) / np.linalg.norm(W))


def theta_objective(W, W0, s, U, V, band_of_layer):
    """Total squared residual sum_l ||W_l - (diag(s_l) W0_b(l) + U_l V_l^T)||_F^2."""
    W = np.asarray(W, dtype=np.float64)
    total = 0.0
    for l in range(W.shape[0]):
        R = W[l] - theta_reconstruct(W0[band_of_layer[l]], s[l], U[l], V[l])
        total += float(np.sum(R * R))
    return total


def decompose_als(W, G: int, r: int, iters: int, band_of_layer=None, trace=None):
    """Alternating least squares over the band-mean start ("Quality (Gemma 4
    31B)", "ALS optimization barely helps": ALS tried as an improvement over
    the mean W0).  The pages name the method, not its steps; the reading here:
    starting from ``decompose`` (mean W0, least-squares s, truncated SVD),
    each iteration updates, in order, each exactly minimising the total
    squared residual over its own block of unknowns with the others fixed:

    1. W0_b[n] = sum_{l in b} s_l[n] (W_l[n] - (U_l V_l^T)[n]) / sum_{l in b} s_l[n]^2
       (the row is kept when every s_l[n] is zero);
    2. s_l[n] = <W_l[n] - (U_l V_l^T)[n], W0_b[n]> / ||W0_b[n]||^2 (1 for a zero row);
    3. U_l V_l^T = truncated SVD of W_l - diag(s_l) W0_b, as in ``decompose``.

    `trace`, if a list, receives the total squared residual after the start
    and after every step.  Returns (W0, s, U, V) like ``decompose``."""
    W = np.asarray(W, dtype=np.float64)
    L, N, K = W.shape
    bands = band_of_layer_contiguous(L, G) if band_of_layer is None else list(band_of_layer)
    W0, s, U, V = decompose(W, G, r, bands)
    if trace is not None:
        trace.append(theta_objective(W, W0, s, U, V, bands))
    for _ in range(iters):
        UV = [U[l] @ V[l].T for l in range(L)]
        for b in range(G):
            members = [l for l in range(L) if bands[l] == b]
            if not members:
                continue
            num = np.zeros((N, K))
            den = np.zeros(N)
            for l in members:
                num += s[l][:, None] * (W[l] - UV[l])
                den += s[l] * s[l]
            keep = den <= 0
            W0[b] = np.where(keep[:, None], W0[b], num / np.where(keep, 1.0, den)[:, None])
        if trace is not None:
            trace.append(theta_objective(W, W0, s, U, V, bands))
        for l in range(L):
            w0 = W0[bands[l]]
            num = np.einsum("nk,nk->n", W[l] - UV[l], w0)
            den = np.einsum("nk,nk->n", w0, w0)
            s[l] = np.where(den > 0, num / np.where(den > 0, den, 1.0), 1.0)
        if trace is not None:
            trace.append(theta_objective(W, W0, s, U, V, bands))
        for l in range(L):
            U[l] = 0.0
            V[l] = 0.0
            if r > 0:
                R = W[l] - s[l][:, None] * W0[bands[l]]
                P, sig, Qt = np.linalg.svd(R, full_matrices=False)
                kk = min(r, sig.shape[0])
                U[l, :, :kk] = P[:, :kk] * sig[:kk]
                V[l, :, :kk] = Qt[:kk].T
        if trace is not None:
            trace.append(theta_objective(W, W0, s, U, V, bands))
    return W0, s, U, V

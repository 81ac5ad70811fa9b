"""Bytes model of a theta bundle and of one forward call.

Theta-bundle size ("Compression" page, "Theta-bundle size: the sharing
headroom"): the shared block W0 is stored once per band and family, the scale s
and the low-rank factors U, V once per layer and family.

Algorithmic bytes of one forward call (what the decode roofline divides by):
W0 (N K), U (N r), V (K r) and s (N) are read once, x (M K) read, y (M N)
written.  "Weight bytes" are the first three parameter terms plus s.
"""
from __future__ import annotations


def dense_bytes(families: dict, num_layers: int, elem_bytes: int = 4) -> int:
    """Dense projection weights of a model: L * sum_f N_f K_f elements."""
    return num_layers * sum(N * K for (N, K) in families.values()) * elem_bytes


def theta_bytes(families: dict, num_layers: int, num_bands: int, rank: int,
                elem_bytes: int = 4) -> int:
    """Theta bundle: G * sum_f N K (W0) + L * sum_f (N + (N + K) r) (s, U, V)."""
    w0 = num_bands * sum(N * K for (N, K) in families.values())
    per_layer = sum(N + (N + K) * rank for (N, K) in families.values())
    return (w0 + num_layers * per_layer) * elem_bytes


def call_weight_bytes(N: int, K: int, r: int, w_bytes: int = 2, s_bytes: int = 4) -> int:
    """Parameter bytes one call streams: W0 + U + V (bf16) + s (fp32)."""
    return (N * K + (N + K) * r) * w_bytes + N * s_bytes


def call_io_bytes(M: int, N: int, K: int, elem_bytes: int = 2) -> int:
    """Activation bytes of one call: x read, y written."""
    return (M * K + M * N) * elem_bytes


def call_flops(M: int, N: int, K: int, r: int) -> int:
    """2MNK (W0 x) + 2MKr (V^T x) + 2MNr (U T)."""
    return 2 * M * N * K + 2 * M * K * r + 2 * M * N * r

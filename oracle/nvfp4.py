"""NVFP4 weight encoding and the theta-bundle forward over an NVFP4-encoded W0.

TEST INFRASTRUCTURE ONLY, like the rest of ``oracle/``: plain numpy fp64,
written from the format's definition, sharing nothing with the CUDA library.

The format ("Compression", section "NVFP4: 3.18x smaller weights"): packed
4-bit weights plus one float8_e4m3fn block scale per 16 elements, 0.5625 bytes
per element.  What the page leaves open is read as follows:

* element code: FP4 E2M1 -- sign bit 3, exponent bits 2..1 (bias 1), one
  mantissa bit; magnitudes 0, 0.5, 1, 1.5, 2, 3, 4, 6 (no infinities, no NaN);
* block: 16 consecutive elements of a row along K (K % 16 == 0); its scale is
  one FP8 E4M3 byte (sign, 4 exponent bits with bias 7, 3 mantissa bits;
  S.1111.111 is NaN, no infinities; largest finite 448);
* one fp32 scale per tensor, as in NVIDIA's two-level NVFP4 layout.  It
  brings the block scales of small weights into E4M3's normal range and adds 4
  bytes per tensor, so the per-element cost stays 0.5625 bytes.  A tensor
  scale of 1 is the one-level reading;
* storage: codes row-major, two per byte, element 2i in the low nibble and
  2i + 1 in the high nibble (N x K/2 bytes); scales row-major (N x K/16);
* quantisation (the page says the weights are quantised at load time but not
  how): tensor scale = max|W| / (6 * 448) rounded to fp32 (the stored
  number, which the block scales are then taken against); block scale = the
  block's max|w| / (6 * tensor scale), rounded to nearest-even E4M3 and
  saturated at 448; code = w / (block scale * tensor scale) rounded to
  nearest-even E2M1 and saturated at +-6; a block whose scale rounds to 0
  gets codes 0.  These divisions are taken in fp64.

Dequantised weight: w = e2m1(code) * e4m3(scale byte) * tensor scale.
"""
from __future__ import annotations

import numpy as np

BLOCK = 16          # elements per E4M3 scale
E2M1_MAX = 6.0
E4M3_MAX = 448.0

# E2M1 magnitudes of codes 0..7: exponent field e = code >> 1, mantissa m = code & 1;
# e == 0 is subnormal (m * 0.5), otherwise (1 + m / 2) * 2^(e - 1).
_E2M1_MAG = np.array([(c & 1) * 0.5 if (c >> 1) == 0 else (1.0 + (c & 1) / 2.0) * 2.0 ** ((c >> 1) - 1)
                      for c in range(8)])
E2M1_VALUES = np.concatenate([_E2M1_MAG, -_E2M1_MAG])  # index = 4-bit code (bit 3 = sign)


def e4m3_decode(b) -> np.ndarray:
    """FP8 E4M3 (fn) bytes -> fp64 values."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b >> 7, -1.0, 1.0)
    e = (b >> 3) & 15
    m = b & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & (m == 7), np.nan, mag)
    return sign * mag


_E4M3_POS = e4m3_decode(np.arange(0x7F))  # finite non-negative values, codes 0x00..0x7E, increasing


def _round_to_grid(v, grid, even):
    """Nearest grid value for each v >= 0 (grid increasing, v within its range),
    ties to the entry whose `even` flag is set; returns grid indices."""
    hi = np.clip(np.searchsorted(grid, v, side="left"), 1, len(grid) - 1)
    lo = hi - 1
    dlo = v - grid[lo]
    dhi = grid[hi] - v
    pick_hi = (dhi < dlo) | ((dhi == dlo) & even[hi])
    return np.where(pick_hi, hi, lo)


def e4m3_encode(x) -> np.ndarray:
    """Non-negative fp64 values -> E4M3 bytes, round to nearest-even,
    saturated at 448."""
    x = np.minimum(np.asarray(x, dtype=np.float64), E4M3_MAX)
    assert np.all(x >= 0)
    idx = _round_to_grid(x, _E4M3_POS, (np.arange(0x7F) & 1) == 0)
    return idx.astype(np.uint8)


def e2m1_encode(v) -> np.ndarray:
    """fp64 values -> E2M1 codes (0..15), round to nearest-even, saturated at
    +-6.  Zero and values that round to zero keep code 0 or 8 by sign."""
    v = np.asarray(v, dtype=np.float64)
    mag = np.minimum(np.abs(v), E2M1_MAX)
    idx = _round_to_grid(mag, _E2M1_MAG, (np.arange(8) & 1) == 0)
    return (idx + np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def pack_codes(codes) -> np.ndarray:
    """N x K codes (0..15) -> N x K/2 bytes, element 2i in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def unpack_codes(packed) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 15
    out[:, 1::2] = p >> 4
    return out


def quantize(W, tensor_scale=None):
    """W (N x K, K % 16 == 0) -> (packed codes N x K/2 uint8, scale bytes
    N x K/16 uint8, tensor scale float)."""
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    assert K % BLOCK == 0, "K must be a multiple of 16"
    if tensor_scale is None:
        amax = float(np.max(np.abs(W))) if W.size else 0.0
        ts32 = float(np.float32(amax / (E2M1_MAX * E4M3_MAX)))
        tensor_scale = ts32 if ts32 > 0 else 1.0  # an all-zero (or vanishing) weight
    blocks = W.reshape(N, K // BLOCK, BLOCK)
    bmax = np.max(np.abs(blocks), axis=2)
    sbytes = e4m3_encode(bmax / (E2M1_MAX * tensor_scale))
    sval = e4m3_decode(sbytes)
    denom = (sval * tensor_scale)[:, :, None]
    q = np.divide(blocks, denom, out=np.zeros_like(blocks), where=denom > 0)
    codes = e2m1_encode(q).reshape(N, K)
    return pack_codes(codes), sbytes, float(tensor_scale)


def dequantize(packed, sbytes, tensor_scale) -> np.ndarray:
    """-> fp64 W (N x K)."""
    codes = unpack_codes(packed)
    N, K = codes.shape
    vals = E2M1_VALUES[codes].reshape(N, K // BLOCK, BLOCK)
    return (vals * e4m3_decode(sbytes)[:, :, None] * tensor_scale).reshape(N, K)


def encoded_bytes(N: int, K: int) -> int:
    """Bytes of an encoded N x K weight without the 4-byte tensor scale."""
    return N * K // 2 + N * K // BLOCK


def forward(x, packed, sbytes, tensor_scale, s, U=None, V=None) -> np.ndarray:
    """y = s (.) (W0 x) + U (V^T x) with W0 the dequantised NVFP4 weight and
    the other operands as given (bf16 tensors or arrays, read exactly), in
    fp64.  x: M x K, s: N, U: N x r, V: K x r; y: M x N."""
    def f64(t):
        if t is None:
            return None
        if hasattr(t, "detach"):
            return t.detach().cpu().double().numpy()
        return np.asarray(t, dtype=np.float64)

    X = f64(x)
    W0 = dequantize(packed, sbytes, tensor_scale)
    y = f64(s)[None, :] * (X @ W0.T)
    Uf, Vf = f64(U), f64(V)
    if Uf is not None and Uf.shape[1] > 0:
        y = y + (X @ Vf) @ Uf.T
    return y

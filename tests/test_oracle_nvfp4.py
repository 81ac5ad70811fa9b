"""Pins of the NVFP4 oracle ("Compression", section "NVFP4: 3.18x smaller
weights": packed 4-bit weights with one float8_e4m3fn scale per 16 elements,
0.5625 bytes per element).  Each test checks the oracle against something
other than itself: torch's float8_e4m3fn codec, a brute-force nearest-value
search, hand-worked blocks, lossless round trips, the rounding error bound,
the page's byte count, and the C forward oracle."""
import os

import numpy as np
import pytest
import torch

import oracle
from oracle import nvfp4

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nvfp4_blocks.txt")


def test_e4m3_decode_matches_torch():
    b = np.arange(256, dtype=np.uint8)
    mine = nvfp4.e4m3_decode(b)
    ref = torch.from_numpy(b.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(mine), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(mine[ok], ref[ok])
    assert np.nanmax(mine) == 448.0


def test_e4m3_encode_matches_torch_rounding():
    """Round to nearest-even on random values over the whole range, on every
    representable value and on every midpoint between neighbours (ties)."""
    rng = np.random.default_rng(0)
    rand = np.abs(rng.standard_normal(20000)) * np.exp2(rng.uniform(-12, 9, 20000))
    grid = nvfp4.e4m3_decode(np.arange(0x7F))
    mids = (grid[:-1] + grid[1:]) / 2
    x = np.minimum(np.concatenate([rand, grid, mids]), 448.0)
    mine = nvfp4.e4m3_encode(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(mine, ref)
    assert nvfp4.e4m3_encode(np.array([1e6]))[0] == 0x7E  # saturated at 448


def _e2m1_brute(v):
    """Nearest of the 8 magnitudes by exhaustive search, ties to the even code."""
    mag = min(abs(v), 6.0)
    best = min(range(8), key=lambda c: (abs(nvfp4.E2M1_VALUES[c] - mag), c & 1))
    return best + (8 if np.signbit(v) else 0)


def test_e2m1_rounding_brute_force():
    rng = np.random.default_rng(1)
    v = np.concatenate([np.arange(-64, 65) / 8.0, rng.uniform(-8, 8, 4000), [-0.0, 0.0, 1e9, -1e9]])
    mine = nvfp4.e2m1_encode(v)
    assert [int(c) for c in mine] == [_e2m1_brute(float(t)) for t in v]


def test_e2m1_table_shape():
    """Two exponent bits with bias 1 and one mantissa bit: a subnormal step of
    0.5 below 1, then each binade [2^(e-1), 2^e) holds two values, so the
    spacing doubles per binade up to 6; codes 8..15 mirror 0..7."""
    m = nvfp4.E2M1_VALUES[:8]
    assert m[0] == 0 and m[1] == 0.5 and m[-1] == 6
    assert np.all(np.diff(m) > 0)
    assert list(np.diff(m)) == [0.5, 0.5, 0.5, 0.5, 1, 1, 2]
    assert np.array_equal(nvfp4.E2M1_VALUES[8:], -m)
    # every magnitude is exact in E4M3, so value * scale stays exact in fp32/bf16
    e4m3 = set(nvfp4.e4m3_decode(np.arange(0x7F)).tolist())
    assert all(float(t) in e4m3 for t in m)


def _golden():
    rows = []
    for line in open(GOLDEN):
        if not line.strip() or line.startswith("#"):
            continue
        vals, packed, scale = (part.split() for part in line.split("|"))
        rows.append((np.array([float(t) for t in vals]), bytes.fromhex("".join(packed)),
                     int(scale[0], 16)))
    return rows


def test_golden_blocks():
    for vals, packed, scale in _golden():
        p, sb, ts = nvfp4.quantize(vals[None, :], tensor_scale=1.0)
        assert ts == 1.0
        assert bytes(p[0]) == packed
        assert int(sb[0, 0]) == scale


def _exact_weight(rng, N, K, ts):
    """A weight NVFP4 holds exactly: random codes and scale bytes, one code
    of magnitude 6 in every block (so the block maximum fixes the scale), and
    one block at the largest scale 448 (so the tensor maximum fixes ts)."""
    codes = rng.integers(0, 16, size=(N, K)).astype(np.uint8)
    nb = K // 16
    codes.reshape(N, nb, 16)[:, :, 0] = rng.choice([7, 15], size=(N, nb))
    sbytes = rng.integers(0x20, 0x7E, size=(N, nb)).astype(np.uint8)
    sbytes[0, 0] = 0x7E
    W = nvfp4.E2M1_VALUES[codes].reshape(N, nb, 16) * nvfp4.e4m3_decode(sbytes)[:, :, None] * ts
    return W.reshape(N, K), nvfp4.pack_codes(codes), sbytes


def test_lossless_round_trip():
    rng = np.random.default_rng(2)
    ts = 2.0 ** -14
    W, packed, sbytes = _exact_weight(rng, 37, 160, ts)
    p, sb, t = nvfp4.quantize(W)
    assert t == ts
    assert np.array_equal(sb, sbytes)
    # a code whose value is 0 encodes as +0 or -0 alike; compare values
    assert np.array_equal(nvfp4.dequantize(p, sb, t), W)
    nz = nvfp4.unpack_codes(packed) & 7 != 0
    assert np.array_equal(nvfp4.unpack_codes(p)[nz], nvfp4.unpack_codes(packed)[nz])


@pytest.mark.parametrize("std", [0.02, 1.0, 300.0])
def test_rounding_error_bound(std):
    """Per element: E2M1's half spacing is at most a quarter of the value
    above 2 and a quarter of the block scale below it, and the block scale's
    rounding can push a value at most 1/16 over 6 into saturation; so
    |w - q(w)| <= |w| / 4 + S / 4 with S the block's dequantised scale."""
    rng = np.random.default_rng(3)
    W = rng.standard_normal((64, 256)) * std
    W[5, 16:32] = 0.0
    p, sb, ts = nvfp4.quantize(W)
    D = nvfp4.dequantize(p, sb, ts)
    S = np.repeat(nvfp4.e4m3_decode(sb) * ts, 16, axis=1)
    assert np.all(np.abs(W - D) <= np.abs(W) / 4 + S / 4 + 1e-300)
    assert np.all(D[5, 16:32] == 0) and sb[5, 1] == 0
    rel = np.linalg.norm(W - D) / np.linalg.norm(W)
    assert 0.02 < rel < 0.2  # 4-bit codes: a few percent to about a tenth


def test_bytes_per_element():
    """0.5 B of packed codes plus one scale byte per 16 elements: 0.5625 B."""
    W = np.random.default_rng(4).standard_normal((96, 1152))
    p, sb, _ = nvfp4.quantize(W)
    assert p.nbytes + sb.nbytes == nvfp4.encoded_bytes(96, 1152)
    assert nvfp4.encoded_bytes(96, 1152) / (96 * 1152) == 0.5625


def test_forward_matches_the_c_oracle_on_an_exact_weight():
    """With a weight NVFP4 holds exactly (and bf16 too: at most 5 significant
    bits), the NVFP4 forward equals the C fp64 forward on that weight."""
    rng = np.random.default_rng(5)
    M, N, K, r = 3, 40, 96, 8
    W, packed, sbytes = _exact_weight(rng, N, K, 2.0 ** -12)
    W0 = torch.tensor(W, dtype=torch.bfloat16)
    assert np.array_equal(W0.double().numpy(), W)
    x = torch.randn(M, K, generator=torch.Generator().manual_seed(6)).to(torch.bfloat16)
    s = torch.rand(N, generator=torch.Generator().manual_seed(7)) + 0.5
    U = (torch.randn(N, r, generator=torch.Generator().manual_seed(8)) * 0.1).to(torch.bfloat16)
    V = (torch.randn(K, r, generator=torch.Generator().manual_seed(9)) * 0.1).to(torch.bfloat16)
    ref = oracle.forward(x, W0, s, U, V)
    got = nvfp4.forward(x, packed, sbytes, 2.0 ** -12, s, U, V)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12 * np.max(np.abs(ref)))
    no_delta = nvfp4.forward(x, packed, sbytes, 2.0 ** -12, s)
    assert np.allclose(no_delta, oracle.forward(x, W0, s, None, None), rtol=1e-12,
                       atol=1e-12 * np.max(np.abs(ref)))

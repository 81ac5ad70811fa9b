"""The library's host NVFP4 encoder (wl_quantize_nvfp4) against the oracle:
codes, block scales and tensor scale bit for bit.  Both take every rounding
decision on the same fp64 quotient, so any difference is a mistake."""
import numpy as np
import pytest

import linear_wl_forward_b200 as wl
from oracle import nvfp4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    wl.lib()


def _same(W, tensor_scale=0.0):
    W = np.asarray(W, dtype=np.float32)
    c, s, t = wl.quantize_nvfp4(W, tensor_scale)
    oc, os_, ot = nvfp4.quantize(W, None if tensor_scale == 0.0 else float(np.float32(tensor_scale)))
    assert t == np.float32(ot)
    assert np.array_equal(s, os_)
    assert np.array_equal(c, oc)
    return c, s, t


@pytest.mark.parametrize("std", [1e-30, 1e-3, 0.02, 1.0, 1e4, 1e30])
def test_random_weights_bit_exact(std):
    rng = np.random.default_rng(int(np.log10(std)) + 40)
    _same(rng.standard_normal((96, 1152)) * std)


def test_heavy_tails_and_empty_blocks():
    rng = np.random.default_rng(1)
    W = rng.standard_cauchy((40, 320)) * 0.01
    W[3] = 0.0
    W[7, 32:48] = -0.0
    W[9, ::17] = 0.0
    _same(W)


def test_ties_and_grid_values_bit_exact():
    """Elements on the E2M1 grid and exactly halfway between grid values,
    under scales that are exact (block maximum 6 times a power of two) and
    block maxima halfway between E4M3 values."""
    rng = np.random.default_rng(2)
    grid = np.array([0, 0.25, 0.5, 0.75, 1, 1.25, 1.5, 1.75, 2, 2.5, 3, 3.5, 4, 5, 6])
    W = rng.choice(grid, size=(64, 512)) * rng.choice([-1.0, 1.0], size=(64, 512))
    W.reshape(64, 32, 16)[:, :, 0] = 6.0
    W = W * np.exp2(rng.integers(-20, 20, size=(64, 1)))
    _same(W, tensor_scale=1.0)
    e4 = nvfp4.e4m3_decode(np.arange(1, 0x7E))
    mids = (e4[:-1] + e4[1:]) / 2
    V = rng.uniform(-1, 1, size=(len(mids), 16)) * mids[:, None]
    V[:, 3] = 6 * mids  # block maximum on an E4M3 tie (exact in fp32 and after / 6)
    assert np.array_equal(np.max(np.abs(V), axis=1) / 6, mids)
    _same(V, tensor_scale=1.0)


def test_explicit_tensor_scales():
    rng = np.random.default_rng(3)
    W = rng.standard_normal((32, 64))
    for ts in (1.0, 0.5, 3e-4, 7.25, 1e-30):
        _same(W, tensor_scale=ts)


def test_zero_and_empty_matrices():
    c, s, t = _same(np.zeros((5, 32)))
    assert t == 1.0 and not c.any() and not s.any()
    c, s, t = wl.quantize_nvfp4(np.zeros((0, 64), np.float32))
    assert c.shape == (0, 32) and s.shape == (0, 4)


def test_argument_errors():
    W = np.ones((4, 32), np.float32)
    with pytest.raises(wl.WLError):
        wl.quantize_nvfp4(np.ones((4, 24), np.float32))  # K % 16 != 0
    with pytest.raises(wl.WLError):
        wl.quantize_nvfp4(W, tensor_scale=-1.0)
    with pytest.raises(wl.WLError):
        wl.quantize_nvfp4(W, tensor_scale=float("inf"))
    bad = W.copy()
    bad[1, 2] = np.nan
    with pytest.raises(wl.WLError):
        wl.quantize_nvfp4(bad)


def test_seeded_nvfp4_draw_is_a_valid_encoding():
    """The NVFP4 W0 draw (random code and scale bytes) is deterministic per
    key and dequantises to finite weights of the bf16 draw's scale."""
    import wl_inputs

    c, s, t = wl_inputs.draw_w0_nvfp4("gemma3_1b", 1, 0, "all", "gate", 64, 1152)
    c2, s2, t2 = wl_inputs.draw_w0_nvfp4("gemma3_1b", 1, 0, "all", "gate", 64, 1152)
    assert (c == c2).all() and (s == s2).all() and t == t2
    assert c.shape == (64, 576) and s.shape == (64, 72)
    W = nvfp4.dequantize(c.numpy(), s.numpy(), t)
    assert np.all(np.isfinite(W)) and 0.005 < W.std() < 0.05

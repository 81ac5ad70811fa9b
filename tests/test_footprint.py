"""Bytes model pinned to the numbers the pages print (CPU only)."""
import json
import os

from linear_wl_forward_b200 import footprint
import wl_inputs

GOLDEN = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")))


def test_dense_projection_bytes_gemma3_1b():
    b = footprint.dense_bytes(wl_inputs.GEMMA3_1B_FAMILIES, wl_inputs.GEMMA3_1B_LAYERS, 4)
    want = GOLDEN["dense_projection_bytes_gemma3_1b_fp32_MB"]["value"]
    assert round(b / 1e6, 2) == want
    assert b == 1_778_909_184


def test_g13_footprint_is_half():
    fam, L = wl_inputs.GEMMA3_1B_FAMILIES, wl_inputs.GEMMA3_1B_LAYERS
    frac = footprint.theta_bytes(fam, L, 13, 4) / footprint.dense_bytes(fam, L)
    g = GOLDEN["footprint_G13_fraction"]
    assert abs(frac - g["value"]) <= g["tolerance"]


def test_passthrough_footprint_exceeds_dense():
    # G = L stores every layer's own W0 plus the delta: above 100%
    fam, L = wl_inputs.GEMMA3_1B_FAMILIES, wl_inputs.GEMMA3_1B_LAYERS
    assert footprint.theta_bytes(fam, L, L, 4) > footprint.dense_bytes(fam, L)


def test_call_bytes_and_flops():
    # gate projection of the Gemma-4-31B shapes at rank 256, M = 1
    N, K, r = 21504, 5376, 256
    wb = footprint.call_weight_bytes(N, K, r)
    assert wb == 2 * (N * K + (N + K) * r) + 4 * N
    assert abs(wb / 1e6 - 245.0) < 0.5
    assert footprint.call_flops(4096, N, K, r) == 2 * 4096 * N * K + 2 * 4096 * K * r + 2 * 4096 * N * r

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


def _gemma4_projections():
    import wl_inputs

    out = []
    for layer in range(wl_inputs.GEMMA4_31B_LAYERS):
        fam = wl_inputs.gemma4_families(wl_inputs.gemma4_layer_type(layer))
        out.extend(fam.values())
    return out


def test_gemma4_projection_count():
    """60 layers x (q, k, v, o, gate, up, down), with no v projection on the
    10 full-attention layers (k = v): the page's 410 projections."""
    assert len(_gemma4_projections()) == GOLDEN["gemma4_31b_projection_count"]["value"]


def test_gemma4_nvfp4_bytes_match_the_page():
    """The page's bf16 total (61.4 GB, rounded) fixes the bytes outside the
    projections (embeddings, norms: bf16 on both sides); with the workload's
    projection shapes at 0.5625 B per element the NVFP4 total must then
    contain the page's 19.295 GB.  Extra projections (a v on full layers) or
    another per-element cost (0.5 B) fall outside."""
    g = GOLDEN["gemma4_31b_weight_bytes_GB"]
    params = sum(N * K for N, K in _gemma4_projections())
    lo_rest = (g["bf16"] - g["bf16_rounding"]) * 1e9 - 2 * params
    hi_rest = (g["bf16"] + g["bf16_rounding"]) * 1e9 - 2 * params
    assert lo_rest > 0
    nv_lo = 0.5625 * params + lo_rest
    nv_hi = 0.5625 * params + hi_rest
    assert nv_lo <= (g["nvfp4"] + g["nvfp4_rounding"]) * 1e9
    assert nv_hi >= (g["nvfp4"] - g["nvfp4_rounding"]) * 1e9


def test_w0_is_nearly_half_of_the_g1_rank32_bundle():
    """G = 1, rank 32, fp32 at the Gemma-3-1B dimensions: W0 (one per family)
    is nearly half the bundle and s is negligible; W0 does not grow with the
    rank.  Counting W0 per layer, or U and V per band, breaks the share."""
    from linear_wl_forward_b200 import footprint
    import wl_inputs

    fam = wl_inputs.GEMMA3_1B_FAMILIES
    L = wl_inputs.GEMMA3_1B_LAYERS
    total = footprint.theta_bytes(fam, L, 1, 32)
    w0 = footprint.theta_bytes(fam, 1, 1, 0) - 4 * sum(N for N, _ in fam.values())
    s_bytes = 4 * L * sum(N for N, _ in fam.values())
    lo, hi = GOLDEN["w0_share_G1_rank32"]["range"]
    assert lo < w0 / total < hi
    assert s_bytes / total < 0.01
    assert footprint.theta_bytes(fam, L, 1, 4) - footprint.theta_bytes(fam, L, 1, 0) < total - w0

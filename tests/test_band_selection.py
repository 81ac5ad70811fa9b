"""Which shared block W0 a layer's call receives (CPU only).

The pages share W0 across the G layers of a band and give equal band sizes
("12 layers per band" for Gemma 4 31B); the reading here is contiguous bands,
band(l) = floor(l * G / L).  Gemma 4 31B has 10 full-attention and 50 sliding
layers; the reading is full iff l % 6 == 5, attention W0 grouped per layer
type, MLP W0 per band.  These tests pin those readings and that the inputs
hand every layer of a band the same W0 tensor (and other bands a different
one)."""
import pytest

import wl_inputs


@pytest.mark.parametrize("L,G", [(26, 13), (26, 1), (26, 26), (60, 5), (12, 4)])
def test_contiguous_bands_equal_and_ordered(L, G):
    bands = [wl_inputs.contiguous_band(l, L, G) for l in range(L)]
    assert bands == sorted(bands)                      # contiguous, in layer order
    assert set(bands) == set(range(G))                 # every band used
    assert all(bands.count(b) == L // G for b in range(G))  # equal sizes (L % G == 0)


def test_gemma3_g13_pairs_and_gemma4_twelve_per_band():
    assert [wl_inputs.contiguous_band(l, 26, 13) for l in range(4)] == [0, 0, 1, 1]
    assert [wl_inputs.contiguous_band(l, 60, 5) for l in (0, 11, 12, 59)] == [0, 0, 1, 4]


def test_gemma4_layer_types():
    types = [wl_inputs.gemma4_layer_type(l) for l in range(60)]
    assert types.count("full") == 10 and types.count("sliding") == 50
    assert [l for l, t in enumerate(types) if t == "full"] == list(range(5, 60, 6))


def _w0(call, fam):
    return next(p.W0 for p in call.projs if p.family == fam)


def test_gemma3_calls_share_w0_within_a_band_only():
    calls = wl_inputs.gemma3_sweep(seed=2, G=13, r=4, M=1, layers=[0, 1, 2])
    by_layer = {}
    for c in calls:
        by_layer.setdefault(c.layer, []).append(c)
    gu = {l: next(c for c in cs if c.projs[0].family == "gate") for l, cs in by_layer.items()}
    assert _w0(gu[0], "gate") is _w0(gu[1], "gate")        # layers 0, 1: band 0
    assert _w0(gu[0], "gate") is not _w0(gu[2], "gate")    # layer 2: band 1
    # the per-layer delta is never shared
    assert gu[0].projs[0].U is not gu[1].projs[0].U


def test_gemma4_w0_grouped_by_layer_type_for_attention_and_by_band_for_mlp():
    # Layers 0..5 are band 0; 4 is sliding, 5 is full.  Shapes are kept by
    # drawing only the smaller families.
    calls = wl_inputs.gemma4_calls(seed=4, r=2, M=1, layers=[0, 4, 5], families=("q", "down"))
    q = {c.layer: _w0(c, "q") for c in calls if any(p.family == "q" for p in c.projs)}
    down = {c.layer: _w0(c, "down") for c in calls if any(p.family == "down" for p in c.projs)}
    assert q[0] is q[4]                    # sliding q of one band: shared
    assert q[5] is not q[0]                # full-attention q: its own block (and shape)
    assert q[5].shape[0] == 16384 and q[0].shape[0] == 8192
    assert down[0] is down[4] is down[5]   # MLP: shared across layer types in a band

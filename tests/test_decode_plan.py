"""Host-side decode planning (no GPU): the choices the decode kernel makes for
the workloads' calls, and the layout invariants the kernel relies on, over a
seeded sweep of shapes.  The plans come from wl_describe_decode_plan, which
runs the library's planner without tensor maps or launches."""
import numpy as np
import pytest

import linear_wl_forward_b200 as wl

SMALL_SMEM = 110 * 1024
MAX_SMEM = 227 * 1024


@pytest.fixture(scope="module", autouse=True)
def _lib():
    wl.lib()


def plan(M, K, projs, sms=148):
    return wl.describe_decode_plan(M, K, projs, sms)


# Gemma-3-1B shapes (hidden 1152, q 1024, k/v 256, MLP 4096), rank 16, M = 1
GEMMA3_CALLS = {
    "qkv": (1152, [(1024, 16), (256, 16), (256, 16)]),
    "o": (1024, [(1152, 16)]),
    "gate_up": (1152, [(4096, 16), (4096, 16)]),
    "down": (4096, [(1152, 16)]),
}


@pytest.mark.parametrize("name", list(GEMMA3_CALLS))
def test_gemma3_calls_form_t_inside_the_stream(name):
    """Every call of the Gemma-3 sweep takes local T fused into the first
    step; all but the down projection run in the compact two-CTA/SM variant.
    The down projection's 128 KB of V rows go to the full-size variant,
    staged, instead of the grid-wide exchange."""
    K, projs = GEMMA3_CALLS[name]
    p = plan(1, K, projs)
    assert p["auto_decode"] == 1
    assert p["t_mode"] == 1 and p["t_fused"] == 1
    assert p["v_stage"] == 1 and p["u_stage"] == 1 and p["v_in_ring"] == 0
    assert p["compact"] == (0 if name == "down" else 1)
    assert p["seg_split"] == (1 if name == "gate_up" else 0)


def test_rank8_down_projection_stages_v():
    """V of 64 KB does not fit the compact variant beside x and a ring level;
    the call must go to the full-size variant with V staged, not to T formed
    element by element on the CUDA cores."""
    p = plan(1, 4096, [(1152, 8)])
    assert p["v_stage"] == 1 and p["compact"] == 0 and p["t_fused"] == 1


def test_gemma4_decode_uses_grid_mode():
    """Rank 256 over K = 5376 (2.75 MB of V per projection) is far beyond any
    CTA's shared memory: partial sums over K slices, three steps of lag, V in
    the ring's last level until they are formed."""
    p = plan(1, 5376, [(21504, 256), (21504, 256)])
    assert p["t_mode"] == 2 and p["lag"] == 3 and p["t_fused"] == 0
    assert p["compact"] == 0 and p["v_in_ring"] == 1
    assert p["grid"] == 148


@pytest.mark.parametrize("M,r,off,fused", [(8, 32, 0, 1), (9, 16, 0, 0), (1, 40, 0, 0), (1, 16, 2, 0),
                                           (1, 24, 0, 1), (4, 8, 0, 1)])
def test_fused_t_conditions(M, r, off, fused):
    """Fused T needs M <= 8, a rank of at most two 16-column tiles, and U, V
    that bulk copies and ldmatrix can read (r % 8 == 0, 16-byte aligned)."""
    p = plan(M, 1152, [(1024, r, off)])
    assert p["t_fused"] == fused
    if off:
        assert p["v_stage"] == 0 and p["u_stage"] == 0


def test_rank_zero_call_has_no_t():
    p = plan(1, 1152, [(4096, 0), (4096, 0)])
    assert p["t_mode"] == 0 and p["v_stage"] == 0 and p["u_stage"] == 0 and p["t_fused"] == 0


@pytest.mark.parametrize("M,rows,expected", [(1, 100000, 1), (4, 43008, 1), (5, 8191, 1), (5, 8192, 0),
                                             (16, 5000, 1), (16, 43008, 0)])
def test_auto_path_rule(M, rows, expected):
    """WL_PATH_AUTO: decode for M <= 4, and for M <= 16 when the call's
    projections total fewer than 8192 output rows."""
    p = plan(M, 1152, [(rows, 16)])
    assert p["auto_decode"] == expected


def test_rejections():
    with pytest.raises(wl.WLError):
        plan(17, 1152, [(100, 8)])  # above WL_DECODE_MAX_M
    with pytest.raises(wl.WLError):
        plan(1, 1156, [(100, 8)])  # K % 8 != 0
    with pytest.raises(wl.WLError):
        plan(1, 1152, [(100, 8)] * 9)  # more than WL_MAX_PROJ projections
    with pytest.raises(wl.WLError):
        plan(1, 1152, [(100, 8)], sms=0)


def _check_invariants(M, K, projs, sms, p):
    rs = [q[1] for q in projs]
    any_r = any(rs)
    aligned = all(r % 8 == 0 and (len(q) < 3 or q[2] % 16 == 0) for q, r in zip(projs, rs) if r)
    blocks = sum((q[0] + 15) // 16 for q in projs)
    assert 1 <= p["grid"] <= min(blocks, sms)
    assert p["smem_bytes"] <= (SMALL_SMEM if p["compact"] else MAX_SMEM)
    assert p["slots"] >= 1 and 1 <= p["slot_chunks"] <= 4
    if p["compact"]:
        assert p["x_smem"] == 1
        if any_r and aligned:
            assert p["v_stage"] == 1  # never T on the CUDA cores in the compact variant
    if p["t_fused"]:
        assert M <= 8 and max(rs) <= 32 and aligned
        assert p["t_mode"] == 1 and p["v_stage"] and p["u_stage"] and not p["v_in_ring"] and p["x_smem"]
    if p["v_in_ring"]:
        assert p["v_stage"] and p["slots"] >= 2 and not p["u_stage"]
    if p["u_stage"] or p["v_stage"]:
        assert any_r and aligned
    assert (p["t_mode"] > 0) == any_r
    assert p["lag"] == (3 if p["t_mode"] == 2 else 0)
    if p["t_mode"] == 1 and aligned:
        # local T over V rows beyond 96 KB only when they are staged
        v_cta = max(K * r * 2 for r in rs if r)
        if v_cta > 96 * 1024 and not p["seg_split"] and len([r for r in rs if r]) == 1:
            assert p["v_stage"] == 1


def test_plan_invariants_over_shapes():
    """A seeded sweep of decode shapes: every plan the planner accepts keeps
    the kernel's shared-memory budget and the combinations it supports."""
    rng = np.random.default_rng(11)
    ranks = [0, 1, 5, 8, 16, 24, 32, 40, 64, 128, 256]
    accepted = 0
    for _ in range(600):
        M = int(rng.integers(1, 17))
        K = int(rng.choice([8, 64, 520, 1024, 1152, 1160, 2056, 4096, 5376, 8192, 21504]))
        P = int(rng.integers(1, 4))
        projs = []
        for _ in range(P):
            N = int(rng.choice([1, 17, 256, 1024, 1152, 3000, 4096, 21504]))
            r = int(rng.choice(ranks))
            off = 2 if rng.random() < 0.1 else 0
            projs.append((N, r, off))
        sms = int(rng.choice([148, 132, 20]))
        try:
            p = plan(M, K, projs, sms)
        except wl.WLError as e:
            assert "unsupported" in str(e).lower(), str(e)
            continue
        accepted += 1
        _check_invariants(M, K, projs, sms, p)
    assert accepted > 500


def _workload_calls():
    import wl_inputs

    for stack in wl_inputs.GEMMA3_1B_STACKS:
        fam = wl_inputs.GEMMA3_1B_FAMILIES
        yield "gemma3", fam[stack[0]][1], [fam[f][0] for f in stack]
    for lt in ("sliding", "full"):
        fam = wl_inputs.gemma4_families(lt)
        for stack in wl_inputs.gemma4_stacks(lt):
            yield f"gemma4_{lt}", fam[stack[0]][1], [fam[f][0] for f in stack]


@pytest.mark.parametrize("M", [1, 2, 4, 8, 9, 16])
@pytest.mark.parametrize("r", [16, 64, 256])
def test_every_workload_call_plans_for_decode(M, r):
    """Every projection stack of the Gemma-3-1B and Gemma-4-31B layers, at
    1-16 tokens and ranks 16-256, is a shape the decode kernel takes (so
    WL_PATH_AUTO never falls back for these), within its invariants."""
    for name, K, Ns in _workload_calls():
        projs = [(N, r) for N in Ns]
        p = plan(M, K, projs)
        _check_invariants(M, K, projs, 148, p)
        if name == "gemma3" and M <= 8 and r <= 32:
            # fused local T, except the down projection (K = 4096) beyond two
            # tokens: its staged x (33-66 KB) no longer fits beside the
            # 128 KB of V rows and a ring level, so it takes grid mode
            fused = K < 4096 or M <= 2
            assert p["t_fused"] == (1 if fused else 0), (name, K, Ns)
            assert p["t_mode"] == (1 if fused else 2), (name, K, Ns)

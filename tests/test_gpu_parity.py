"""GPU parity: every kernel path against the fp64 oracle, through the C ABI,
at small ragged sizes (several tiles plus a tail), at the workloads' full
sizes, and on the edge cases."""
import numpy as np
import pytest
import torch

import linear_wl_forward_b200 as wl
import oracle
import wl_inputs
from gpu_util import check_call, compare, run, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    wl.lib()


# ------------------------------------------------------------ tiny band ----
@pytest.mark.parametrize("path", ["auto", "decode", "gemm"])
def test_tiny_band_both_layers(path):
    """G=2 layers sharing one W0 (256 x 128), rank 4, x 4 x 128, seed 0."""
    for call in wl_inputs.tiny_band(0):
        check_call(call, path)


# ---------------------------------------------------------- ragged cases ---
DECODE_CASES = [(1, 1, 8, 0), (1, 37, 24, 5), (2, 300, 1000, 16), (3, 513, 1032, 64),
                (4, 257, 2056, 256), (1, 2000, 3080, 8), (4, 129, 64, 1024), (2, 64, 8, 3),
                (8, 700, 4104, 24), (13, 333, 520, 256), (16, 2048, 5376, 256), (9, 17, 16, 7),
                (16, 40, 8, 0), (5, 4000, 136, 1000),
                # T formed inside the first step (rank <= 32, M <= 8): two-block
                # CTAs with a ragged K, V of 128 KB (full-size variant), a rank
                # of one and a half 16-column tiles with V above 96 KB
                (5, 3000, 1160, 32), (1, 1152, 4096, 16), (7, 700, 2056, 24), (1, 1152, 4096, 8)]
GEMM_CASES = [(1, 37, 24, 5), (5, 300, 200, 16), (130, 513, 1000, 64), (257, 255, 136, 72),
              (64, 1024, 520, 256), (200, 77, 64, 0), (129, 600, 2056, 4), (16, 256, 256, 1024),
              (300, 1, 8, 8)]


@pytest.mark.parametrize("M,N,K,r", DECODE_CASES)
def test_decode_ragged(M, N, K, r):
    check_call(wl_inputs.random_case(11 + M + N + K + r, M, N, K, r), "decode")


@pytest.mark.parametrize("M,N,K,r", GEMM_CASES)
def test_gemm_ragged(M, N, K, r):
    check_call(wl_inputs.random_case(23 + M + N + K + r, M, N, K, r), "gemm")


@pytest.mark.parametrize("path,M", [("decode", 3), ("decode", 11), ("gemm", 70)])
def test_stacked_mixed_ranks(path, M):
    call = wl_inputs.random_case(5, M, [300, 64, 1000], 512, [16, 0, 40], P=3)
    check_call(call, path)


@pytest.mark.parametrize("path,M", [("decode", 2), ("decode", 16), ("gemm", 33)])
def test_stacked_max_projections(path, M):
    Ns = [40, 8, 130, 256, 17, 300, 64, 9]
    rs = [8, 16, 0, 64, 3, 32, 256, 8]
    call = wl_inputs.random_case(6, M, Ns, 256, rs, P=wl.MAX_PROJ)
    check_call(call, path)


def test_deterministic_repeat():
    for path, M in (("decode", 4), ("decode", 16), ("gemm", 150)):
        call = wl_inputs.random_case(8, M, 700, 1544, 64)
        xd, pd = to_dev(call)
        a = run(call, path, xd, pd)[0]
        b = run(call, path, xd, pd)[0]
        assert np.array_equal(a, b)


def test_paths_agree_at_small_m():
    call = wl_inputs.random_case(9, 4, 1000, 2048, 64)
    yd = run(call, "decode")[0]
    yg = run(call, "gemm")[0]
    compare(yd, yg, "decode vs gemm")


# ------------------------------------------------------------ edge cases ---
def test_empty_inputs_are_noops():
    x = torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda")
    W0 = torch.zeros(16, 64, dtype=torch.bfloat16, device="cuda")
    s = torch.ones(16, device="cuda")
    y = wl.linear_forward(x, W0, s, None, None)
    assert y.shape == (0, 16)
    x1 = torch.ones(2, 64, dtype=torch.bfloat16, device="cuda")
    y0 = wl.linear_forward(x1, torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda"),
                           torch.ones(0, device="cuda"), None, None)
    assert y0.shape == (2, 0)


def test_k_zero_gives_zeros():
    x = torch.zeros(3, 0, dtype=torch.bfloat16, device="cuda")
    W0 = torch.zeros(5, 0, dtype=torch.bfloat16, device="cuda")
    y = torch.full((3, 5), 7.0, dtype=torch.bfloat16, device="cuda")
    wl.linear_forward(x, W0, torch.ones(5, device="cuda"), None, None, y=y)
    torch.cuda.synchronize()
    assert torch.all(y == 0)


def test_exact_small_integers_bit_exact():
    """Small integers are exact in bf16 and fp32 sums: both paths must equal
    the oracle bit for bit."""
    rng = np.random.default_rng(3)
    M, N, K, r = 4, 96, 64, 8
    x = torch.tensor(rng.integers(-1, 2, (M, K)), dtype=torch.bfloat16)
    W0 = torch.tensor(rng.integers(-2, 3, (N, K)), dtype=torch.bfloat16)
    s = torch.tensor(rng.integers(-2, 3, (N,)) * 0.5, dtype=torch.float32)
    U = torch.tensor(rng.integers(-1, 2, (N, r)), dtype=torch.bfloat16)
    V = torch.tensor(rng.integers(-1, 2, (K, r)), dtype=torch.bfloat16)
    ref = oracle.forward(x, W0, s, U, V)
    assert np.max(np.abs(ref)) < 128  # half-integers below 128 are exact in bf16
    for path in ("decode", "gemm"):
        y = wl.stacked_forward(x.cuda(), [(W0.cuda(), s.cuda(), U.cuda(), V.cuda())], path=path)[0]
        assert np.array_equal(y.float().cpu().numpy(), ref), path


def test_wait_timeout_is_reported():
    """A device wait that nobody releases gives up and reports WL_ERR_TIMEOUT;
    the context stays usable."""
    wl.wait_probe(2_000_000)
    assert wl.last_device_status() == 5
    assert wl.last_device_status() == 0
    check_call(wl_inputs.random_case(1, 1, 64, 64, 8), "decode")


def test_bad_arguments_raise():
    x = torch.ones(2, 12, dtype=torch.bfloat16, device="cuda")
    W0 = torch.ones(4, 12, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wl.WLError) as e:
        wl.linear_forward(x, W0, torch.ones(4, device="cuda"), None, None)
    assert e.value.code == 2
    x = torch.ones(wl.DECODE_MAX_M + 1, 16, dtype=torch.bfloat16, device="cuda")
    W0 = torch.ones(4, 16, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(wl.WLError):
        wl.linear_forward(x, W0, torch.ones(4, device="cuda"), None, None, path="decode")


# ------------------------------------------------------ workload shapes ----
def test_gemma3_1b_decode_layer():
    """Gemma-3-1B shapes, 13 bands of 2 layers, rank 16, M = 1: every
    projection stack of layers 0 and 1 (they share W0)."""
    for call in wl_inputs.gemma3_sweep(seed=2, G=13, r=16, M=1, layers=[0, 1]):
        check_call(call)


@pytest.mark.parametrize("M", [1, 8, 64])
def test_gemma3_1b_stacked_g1_rank64(M):
    for call in wl_inputs.gemma3_sweep(seed=3, G=1, r=64, M=M, layers=[0]):
        check_call(call)


@pytest.mark.parametrize("M", [1, 16])
@pytest.mark.parametrize("layer", [0, 5])
def test_gemma4_31b_decode(M, layer):
    """Gemma-4-31B shapes at rank 256: a sliding layer (0) and a full-attention
    layer (5), every stack."""
    for call in wl_inputs.gemma4_calls(seed=4, r=256, M=M, layers=[layer]):
        check_call(call)


def test_gemma4_31b_prefill_sampled_rows():
    """M = 4096 prefill at full size; outputs checked on 16 seeded random token
    rows plus the first and last row (the oracle would take minutes for all)."""
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([[0, 4095], rng.choice(4096, 16, replace=False)]))
    for layer in (0, 5):
        for call in wl_inputs.gemma4_calls(seed=5, r=256, M=4096, layers=[layer]):
            if layer == 5 and call.projs[0].family in ("gate", "down"):
                continue  # MLP shapes already covered by layer 0
            check_call(call, rows=rows)


@pytest.mark.gpu
def test_prepared_matches_stacked():
    """A prepared call (checks and marshalling done once, then issued twice)
    gives the same bits as stacked_forward on the same inputs."""
    import torch

    for M in (1, 12, 40):
        call = wl_inputs.random_case(31 + M, M, [300, 64], 520, [16, 8], P=2)
        xd, pd = to_dev(call)
        ref = [y.cpu() for y in wl.stacked_forward(xd, pd)]
        prep = wl.prepare_stacked(xd, pd)
        for _ in range(2):
            got = [y.cpu() for y in prep()]
            torch.cuda.synchronize()
            for a, b in zip(ref, got):
                assert torch.equal(a, b)
        assert wl.last_device_status() == 0


@pytest.mark.parametrize("M,ranks", [(1, [0, 16, 32]), (2, [0, 16]), (8, [16, 0, 8])])
def test_stacked_fused_t_with_rank_zero_projection(M, ranks):
    """T formed inside the first step, in a stacked call where some CTAs' rows
    have no delta (they stage no V or U rows) and the ranks need one or two
    16-column tiles of T."""
    plan = wl.describe_decode_plan(M, 520, [(n, r) for n, r in zip([300, 200, 40], ranks)])
    assert plan["t_fused"] == 1
    call = wl_inputs.random_case(60 + M, M, [300, 200, 40][:len(ranks)], 520, ranks, P=len(ranks))
    check_call(call, "decode")


# ------------------------------------------------------- L2 prefetch hint ---
@pytest.mark.parametrize("path,M", [("decode", 1), ("decode", 8), ("gemm", 16), ("gemm", 130)])
def test_prefetch_leaves_results_unchanged(path, M):
    """wl_stacked_forward_prefetch only pulls ranges into L2: the outputs are
    bit-identical to the call without it and match the oracle.  The ranges
    include the next call's weights, an odd-sized range at an odd address, an
    empty one, and the call's own output buffer."""
    call = wl_inputs.random_case(31 + M, M, [700, 129], 1032, [16, 8], P=2)
    nxt = wl_inputs.random_case(32 + M, 1, 2000, 1152, 16)
    xd, pd = to_dev(call)
    _, npd = to_dev(nxt)
    base = wl.stacked_forward(xd, pd, path=path)
    torch.cuda.synchronize()
    ys = [torch.empty_like(y) for y in base]
    odd = torch.empty(4099, dtype=torch.uint8, device="cuda")
    pf = [t for t in npd[0]] + [(odd.data_ptr() + 3, 4093), (odd.data_ptr(), 0), ys[0]]
    for _ in range(2):
        wl.stacked_forward(xd, pd, ys=ys, path=path, prefetch=pf)
    torch.cuda.synchronize()
    assert wl.last_device_status() == 0
    for p, y, yb in zip(call.projs, ys, base):
        assert torch.equal(y, yb)
        ref = oracle.forward(call.x, p.W0, p.s, p.U, p.V)
        compare(y.double().cpu().numpy(), ref, f"prefetch {path} M={M}")

"""GPU parity of the row-stream decode kernel (WL_PATH_ROWS) against the fp64
oracle: ragged shapes (K not a multiple of the 32-column k-group, rows past a
16-row block, one to four blocks per CTA, clusters of 1, 2 and 4 CTAs along
K), stacked calls, the Gemma-3-1B projection stacks, the L2 prefetch, and
calls the kernel declines."""
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


ROWS_CASES = [(1, 1, 8, 0), (1, 37, 24, 8), (2, 300, 1000, 16), (3, 513, 1032, 64), (1, 2000, 3080, 8),
              (8, 700, 4104, 24), (13, 333, 520, 64), (16, 64, 8, 0), (5, 1000, 136, 40), (9, 17, 16, 16),
              (16, 2048, 1160, 32), (1, 1152, 4096, 16), (4, 4096, 1152, 16), (1, 9000, 264, 8),
              (2, 160, 72, 56), (7, 48, 2056, 0)]


@pytest.mark.parametrize("M,N,K,r", ROWS_CASES)
def test_rows_ragged(M, N, K, r):
    plan = wl.describe_rows_plan(M, K, [(N, r)])
    assert plan["grid"] <= 148 and plan["nb_max"] <= 4
    check_call(wl_inputs.random_case(71 + M + N + K + r, M, N, K, r), "rows")


def test_rows_clusters_of_each_size():
    """The planner's cluster sizes 1, 2 and 4 all occur among these calls and
    each matches the oracle."""
    seen = set()
    for M, N, K, r in [(1, 6000, 1152, 16), (1, 3000, 1152, 16), (2, 600, 2048, 16), (1, 600, 8192, 16)]:
        seen.add(wl.describe_rows_plan(M, K, [(N, r)])["cluster"])
        check_call(wl_inputs.random_case(90 + N, M, N, K, r), "rows")
    assert seen == {1, 2, 4}, seen


@pytest.mark.parametrize("M", [1, 3, 11])
def test_rows_stacked_mixed_ranks(M):
    check_call(wl_inputs.random_case(5, M, [300, 64, 1000], 512, [16, 0, 40], P=3), "rows")


def test_rows_stacked_max_projections():
    Ns = [40, 8, 130, 256, 17, 300, 64, 9]
    rs = [8, 16, 0, 64, 8, 32, 64, 8]
    check_call(wl_inputs.random_case(6, 2, Ns, 256, rs, P=wl.MAX_PROJ), "rows")


@pytest.mark.parametrize("M", [1, 8, 16])
def test_rows_gemma3_1b_layer(M):
    """Every Gemma-3-1B projection stack (q/k/v, o, gate/up, down) of layers 0
    and 1 (one shared W0), rank 16."""
    for call in wl_inputs.gemma3_sweep(seed=2, G=13, r=16, M=M, layers=[0, 1]):
        shapes = [(p.N, p.r) for p in call.projs]
        try:
            wl.describe_rows_plan(M, call.projs[0].K, shapes)
        except wl.WLError:
            # 8 or 16 tokens of the 8192-row gate/up stack need more shared memory
            # than two CTAs per SM allow: that call takes another kernel
            assert M >= 8 and [p.family for p in call.projs] == ["gate", "up"]
            continue
        check_call(call, "rows")


def test_rows_deterministic():
    """Repeat calls give identical bits."""
    call = wl_inputs.random_case(8, 4, 700, 1544, 64)
    xd, pd = to_dev(call)
    a = run(call, "rows", xd, pd)[0]
    b = run(call, "rows", xd, pd)[0]
    assert np.array_equal(a, b)


@pytest.mark.parametrize("M,N,K,r,x_zero,cluster", [(5, 200, 1000, 16, 0.6, 1), (2, 600, 8192, 16, 0.95, 4),
                                                   (3, 300, 8192, 24, 0.95, 4)])
def test_rows_bit_exact_on_small_integers(M, N, K, r, x_zero, cluster):
    """Inputs in {-1, 0, 1} (x sparse enough that every sum stays small) and
    half-integer scales: every partial sum is exact in fp32 and every y is a
    bf16 value, so the kernel -- without clusters and with the cluster's
    sums over distributed shared memory -- must equal the oracle bit for bit."""
    assert wl.describe_rows_plan(M, K, [(N, r)])["cluster"] == cluster
    rng = np.random.default_rng(4)

    def draw(shape, p0):  # -1, 0, 1 with P(0) = p0
        return torch.tensor(rng.choice([-1, 0, 1], size=shape, p=[(1 - p0) / 2, p0, (1 - p0) / 2]),
                            dtype=torch.bfloat16)

    x, W0, U, V = draw((M, K), x_zero), draw((N, K), 0.6), draw((N, r), 0.5), draw((K, r), 0.6)
    s = torch.tensor(rng.integers(-2, 3, (N,)) * 0.5, dtype=torch.float32)
    ref = oracle.forward(x, W0, s, U, V)
    assert np.all(ref == np.round(ref * 2) / 2) and np.max(np.abs(ref)) < 2 ** 20
    assert np.array_equal(torch.tensor(ref).to(torch.bfloat16).double().numpy(), ref)
    y = wl.stacked_forward(x.cuda(), [(W0.cuda(), s.cuda(), U.cuda(), V.cuda())], path="rows")[0]
    assert np.array_equal(y.float().cpu().numpy(), ref)


@pytest.mark.parametrize("M", [1, 8])
def test_rows_prefetch_leaves_results_unchanged(M):
    call = wl_inputs.random_case(33 + M, M, [700, 129], 1032, [16, 8], P=2)
    nxt = wl_inputs.random_case(34 + M, 1, 2000, 1152, 16)
    xd, pd = to_dev(call)
    _, npd = to_dev(nxt)
    base = wl.stacked_forward(xd, pd, path="rows")
    ys = [torch.empty_like(y) for y in base]
    wl.stacked_forward(xd, pd, ys=ys, path="rows", prefetch=list(npd[0]) + [ys[1]])
    torch.cuda.synchronize()
    assert wl.last_device_status() == 0
    for p, y, yb in zip(call.projs, ys, base):
        assert torch.equal(y, yb)
        compare(y.double().cpu().numpy(), oracle.forward(call.x, p.W0, p.s, p.U, p.V), "rows prefetch")


@pytest.mark.parametrize("M,N,K,r", [(1, 64, 64, 12), (1, 64, 64, 72), (1, 64 * 16 * 148 * 4 + 16, 64, 8)])
def test_rows_declines_what_it_does_not_fit(M, N, K, r):
    """Odd ranks, ranks above 64 and calls of more than four blocks per SM
    are declined before any launch (WL_ERR_UNSUPPORTED); the automatic path
    still serves them."""
    call = wl_inputs.random_case(3, M, N, K, r) if N < 100000 else None
    if call is None:
        with pytest.raises(wl.WLError) as e:
            wl.describe_rows_plan(M, K, [(N, r)])
        assert e.value.code == 3
        return
    xd, pd = to_dev(call)
    with pytest.raises(wl.WLError) as e:
        wl.stacked_forward(xd, pd, path="rows")
    assert e.value.code == 3
    check_call(call, "auto")

"""The forward kernels' own bounded waits, made to give up: with a wait limit
of 1 ns (wl_set_wait_limit) a call's waits may expire; such a call reports
WL_ERR_TIMEOUT through wl_last_device_status() instead of hanging, a call
that does not report it is correct, the status read clears the grid-wide
counts a call that gave up leaves set, and the next call at the default
limit is correct again.  Nothing here faults or
hangs a GPU: every wait is bounded, and the kernels let their copies in
flight land before their CTAs exit."""
import pytest
import torch

import linear_wl_forward_b200 as wl
import oracle
import wl_inputs
from gpu_util import check_call, compare, to_dev

pytestmark = pytest.mark.gpu

TIMEOUT = 5


@pytest.fixture(autouse=True)
def _restore_limit():
    assert torch.cuda.is_available()
    assert wl.last_device_status() == 0
    yield
    wl.set_wait_limit(0)
    wl.last_device_status()


def _short_limit_calls(call, path, tries=20):
    """Issues the call `tries` times with a 1 ns wait limit: each call either
    gives up (WL_ERR_TIMEOUT) or is correct, never silently wrong.  Returns
    the statuses."""
    xd, pd = to_dev(call)
    refs = [oracle.forward(call.x, p.W0, p.s, p.U, p.V) for p in call.projs]
    wl.set_wait_limit(1)
    seen = []
    try:
        for _ in range(tries):
            ys = [torch.full((call.x.shape[0], p.N), float("nan"), dtype=torch.bfloat16, device="cuda")
                  for p in call.projs]
            wl.stacked_forward(xd, pd, ys=ys, path=path)
            st = wl.last_device_status()
            assert st in (0, TIMEOUT), st
            seen.append(st)
            if st == 0:
                for y, ref in zip(ys, refs):
                    compare(y.double().cpu().numpy(), ref, f"{path} under a 1 ns wait limit")
    finally:
        wl.set_wait_limit(0)
    assert wl.last_device_status() == 0  # the read cleared it
    return seen


@pytest.mark.parametrize("path,case,mode,must_expire", [
    # decode kernel, T by the grid-wide exchange (two counts every CTA waits
    # on: all but the last CTA to arrive give up)
    ("decode", (4, 1000, 2056, 64), "grid", True),
    # decode kernel, local T (ring and staged-V waits only)
    ("decode", (1, 3000, 1032, 16), "local", False),
    # row-stream kernel (its copies are requested long before its waits, so
    # they rarely expire even at 1 ns)
    ("rows", (1, 1152, 4096, 16), None, False),
    # tensor-core GEMM, swap mode with K ranges summed by the last CTA to
    # arrive (the pipeline's first waits expire before the first tiles land)
    ("gemm", (8, 2048, 5376, 256), "swap", True),
    # tensor-core GEMM, 128-row x tiles
    ("gemm", (200, 600, 2056, 64), None, True),
])
def test_short_wait_limit_gives_up_or_is_correct(path, case, mode, must_expire):
    M, N, K, r = case
    if path == "decode":
        plan = wl.describe_decode_plan(M, K, [(N, r)])
        assert plan["t_mode"] == (2 if mode == "grid" else 1)
    call = wl_inputs.random_case(400 + M + N, M, N, K, r)
    seen = _short_limit_calls(call, path)
    if must_expire:
        assert TIMEOUT in seen, seen
    # at the default limit, after the status read cleared what the calls that
    # gave up left behind, the same call and a second one are correct
    check_call(call, path)
    check_call(wl_inputs.random_case(401 + M + N, M, N, K, r), path)


def test_nvfp4_ring_short_wait_limit_gives_up_or_is_correct():
    """The NVFP4 ring stream's slot waits (consumers on landed copies, the
    producer on freed slots) at a 1 ns limit: each call gives up or is
    correct; blocks split between CTAs leave their counters set when a call
    gives up, which the status read clears, and the next call is correct."""
    from oracle import nvfp4

    M, Ns, K, rs = 2, [700, 2000], 16384, [256, 8]
    assert wl.describe_nvfp4_plan(M, K, list(zip(Ns, rs)))["ring"] == 1
    host, projs = [], []
    for i, (N, r) in enumerate(zip(Ns, rs)):
        codes, scales, ts = wl_inputs.draw_w0_nvfp4("fp4timeout", 1, 0, "all", f"f{i}", N, K)
        s, U, V = wl_inputs.draw_delta("fp4timeout", 1, i, f"f{i}", N, K, r)
        host.append((codes, scales, ts, s, U, V))
        projs.append((codes.cuda(), scales.cuda(), ts, s.cuda(), U.cuda(), V.cuda()))
    x = wl_inputs.draw_x("fp4timeout", 1, M, K)
    refs = [nvfp4.forward(x, c.numpy(), sc.numpy(), ts, s, U, V) for (c, sc, ts, s, U, V) in host]
    xd = x.cuda()
    wl.set_wait_limit(1)
    seen = []
    try:
        for _ in range(20):
            ys = [torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda") for N in Ns]
            wl.stacked_forward_nvfp4(xd, projs, ys=ys)
            st = wl.last_device_status()
            assert st in (0, TIMEOUT), st
            seen.append(st)
            if st == 0:
                for y, ref in zip(ys, refs):
                    compare(y.double().cpu().numpy(), ref, "nvfp4 ring under a 1 ns wait limit")
    finally:
        wl.set_wait_limit(0)
    assert wl.last_device_status() == 0
    for _ in range(2):
        ys = wl.stacked_forward_nvfp4(xd, projs)
        assert wl.last_device_status() == 0
        for y, ref in zip(ys, refs):
            compare(y.double().cpu().numpy(), ref, "nvfp4 ring after the time-outs")

"""The forward kernels' own bounded waits, made to give up: with a wait limit
of a few nanoseconds (wl_set_wait_limit) the waits of a call expire, the call
reports WL_ERR_TIMEOUT through wl_last_device_status() instead of hanging, the
status read clears the grid-wide counts a call that gave up leaves set, and
the next call at the default limit is correct again.  Nothing here faults or
hangs a GPU: every wait is bounded, and the kernels let their copies in
flight land before their CTAs exit."""
import pytest
import torch

import linear_wl_forward_b200 as wl
import wl_inputs
from gpu_util import check_call, to_dev

pytestmark = pytest.mark.gpu

TIMEOUT = 5


@pytest.fixture(autouse=True)
def _restore_limit():
    assert torch.cuda.is_available()
    assert wl.last_device_status() == 0
    yield
    wl.set_wait_limit(0)
    wl.last_device_status()


def _gives_up(call, path, tries=40):
    """Issues the call with a 1 ns wait limit until one of its waits gives up."""
    xd, pd = to_dev(call)
    wl.set_wait_limit(1)
    seen = []
    for _ in range(tries):
        wl.stacked_forward(xd, pd, path=path)
        st = wl.last_device_status()
        seen.append(st)
        if st == TIMEOUT:
            break
    wl.set_wait_limit(0)
    assert TIMEOUT in seen, seen
    assert set(seen) <= {0, TIMEOUT}, seen
    assert wl.last_device_status() == 0  # the read cleared it


@pytest.mark.parametrize("path,case,mode", [
    # decode kernel, T by the grid-wide exchange (two counts every CTA waits on)
    ("decode", (4, 1000, 2056, 64), "grid"),
    # decode kernel, local T (ring and staged-V waits only)
    ("decode", (1, 3000, 1032, 16), "local"),
    # row-stream kernel (the staged V / U wait, inside 4-CTA clusters)
    ("rows", (1, 1152, 4096, 16), None),
    # tensor-core GEMM, swap mode with K ranges summed by the last CTA to arrive
    ("gemm", (8, 2048, 5376, 256), "swap"),
    # tensor-core GEMM, 128-row x tiles
    ("gemm", (200, 600, 2056, 64), None),
])
def test_wait_gives_up_and_the_next_call_is_correct(path, case, mode):
    M, N, K, r = case
    if path == "decode":
        plan = wl.describe_decode_plan(M, K, [(N, r)])
        assert plan["t_mode"] == (2 if mode == "grid" else 1)
    call = wl_inputs.random_case(400 + M + N, M, N, K, r)
    _gives_up(call, path)
    check_call(call, path)
    # a second call of the same shape, after the counts were cleared
    check_call(wl_inputs.random_case(401 + M + N, M, N, K, r), path)

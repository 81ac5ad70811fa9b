"""The allocation-free decode entry point (wl_linear_forward_noalloc).

It serves callers that cannot allocate device memory while they run (code
inside a pre-planned memory arena, or under a hard memory budget): its scratch
is a fixed array in the library's device image instead of the growable pool of
wl_linear_forward.  This test calls it through the C ABI twice in a row, with
different shapes so stale contents of the shared array would show, and checks
each output against wl_linear_forward's within the parity tolerance.  It lives
in its own file, collected last, and does not rely on any earlier test.
Each output is also checked against the fp64 oracle, and the array's own
status word (wl_noalloc_last_status) must read WL_OK.
"""
import ctypes

import pytest
import torch

import linear_wl_forward_b200 as wl
import oracle
import wl_inputs
from gpu_util import FROB_TOL, MAX_TOL, compare

pytestmark = pytest.mark.gpu


def _fn():
    fn = wl.lib().wl_linear_forward_noalloc
    fn.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_int] * 4 + [ctypes.c_void_p]
    fn.restype = ctypes.c_int
    return fn


def _dev(case):
    p = case.projs[0]
    return (case.x.cuda(), p.W0.cuda(), p.s.cuda(), p.U.cuda() if p.r else None,
            p.V.cuda() if p.r else None)


def test_noalloc_matches_linear_forward_on_two_calls():
    """Two grid-mode calls in a row (V^T x exchanged through the array, with
    different grids), so the second runs on the partial sums and counts the
    first left in the shared array."""
    assert torch.cuda.is_available()
    fn = _fn()
    status = wl.lib().wl_noalloc_last_status
    status.argtypes = [ctypes.c_void_p]
    status.restype = ctypes.c_int
    stream = torch.cuda.current_stream().cuda_stream
    cases = [wl_inputs.random_case(41, 4, 1000, 2056, 64),    # M=4, rank 64: 63 CTAs
             wl_inputs.random_case(42, 2, 1500, 3000, 256)]   # then M=2, rank 256: 94 CTAs
    grids = set()
    for case in cases:
        x, W0, s, U, V = _dev(case)
        M, K = x.shape
        N, r = W0.shape[0], (0 if U is None else U.shape[1])
        plan = wl.describe_decode_plan(M, K, [(N, r)])
        assert plan["t_mode"] == 2  # the grid-wide exchange runs through the shared array
        grids.add(plan["grid"])
        y_ref = wl.linear_forward(x, W0, s, U, V)
        y = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        rc = fn(x.data_ptr(), W0.data_ptr(), s.data_ptr(), U.data_ptr() if r else None,
                V.data_ptr() if r else None, y.data_ptr(), M, N, K, r, stream)
        assert rc == 0, wl.STATUS.get(rc, rc)
        assert status(stream) == 0
        torch.cuda.synchronize()
        got = y.double().cpu().numpy()
        compare(got, y_ref.double().cpu().numpy(), "noalloc vs linear_forward")
        p = case.projs[0]
        compare(got, oracle.forward(case.x, p.W0, p.s, p.U, p.V), "noalloc vs oracle")
    assert len(grids) == 2
    assert MAX_TOL == 2e-2 and FROB_TOL == 5e-3


def test_noalloc_rejects_unsupported_shapes_on_the_host():
    fn = _fn()
    fake = 0x10000  # 16-byte aligned, never dereferenced: both are rejected before any launch
    assert fn(fake, fake, fake, fake, fake, fake, wl.DECODE_MAX_M + 1, 64, 64, 8, None) == 3
    assert fn(fake, fake, fake, fake, fake, fake, 1, 64, 64, wl.MAX_RANK + 1, None) == 3

"""GPU parity of the persistent ring decode path (WL_PATH_RING: a V^T x launch,
then one CTA per SM streaming the call's 16-row x 512-column weight tiles,
the work split evenly over the SMs) against the fp64 oracle: ragged shapes
(K not a multiple of the 32-column group or of the 512-column stage, rows
past a 16-row block, blocks split between CTAs, one block over many CTAs),
every rank class the ring takes, one to eight tokens, stacked calls, a full
Gemma-4-31B gate/up stack, and the calls it declines."""
import numpy as np
import pytest
import torch

import linear_wl_forward_b200 as wl
import wl_inputs
from gpu_util import check_call, run, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    wl.lib()


RING_CASES = [(1, 1, 8, 0), (1, 37, 1000, 8), (2, 300, 1032, 16), (3, 513, 4096, 64), (8, 700, 5376, 256),
              (5, 16, 21504, 24), (1, 2000, 520, 0), (4, 64, 8, 8), (7, 1000, 2056, 40)]


@pytest.mark.parametrize("M,N,K,r", RING_CASES)
def test_ring_ragged(M, N, K, r):
    check_call(wl_inputs.random_case(301 + M + N + K + r, M, N, K, r), "ring")


@pytest.mark.parametrize("M", [1, 6])
def test_ring_stacked_mixed_ranks(M):
    check_call(wl_inputs.random_case(31, M, [300, 64, 1000], 2048, [16, 0, 40], P=3), "ring")


def test_ring_gemma4_gate_up():
    """The Gemma-4-31B gate/up stack (2 x 21504 x 5376, rank 256), one token."""
    check_call(wl_inputs.random_case(32, 1, [21504, 21504], 5376, [256, 256], P=2), "ring")


def test_ring_deterministic():
    call = wl_inputs.random_case(33, 2, [3000, 3000], 4096, [64, 64], P=2)
    xd, pd = to_dev(call)
    a = run(call, "ring", xd, pd)
    b = run(call, "ring", xd, pd)
    assert all(np.array_equal(p, q) for p, q in zip(a, b))


@pytest.mark.parametrize("M,N,K,r", [(9, 64, 64, 8), (1, 64, 64, 12), (1, 64, 64, 264)])
def test_ring_declines_what_it_does_not_take(M, N, K, r):
    """More than 8 tokens, odd ranks and ranks above 256 are declined before
    any launch (WL_ERR_UNSUPPORTED)."""
    call = wl_inputs.random_case(34, M, N, K, r)
    xd, pd = to_dev(call)
    with pytest.raises(wl.WLError) as e:
        wl.stacked_forward(xd, pd, path="ring")
    assert e.value.code == 3

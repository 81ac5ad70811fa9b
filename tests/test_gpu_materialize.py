"""GPU parity of the dense-weight rebuild W_eff = diag(s) W0 + U V^T (the
precompute-outside form of "Override the graph build", step 5) against the
fp64 oracle, and of the dense forward it feeds."""
import numpy as np
import pytest
import torch

import linear_wl_forward_b200 as wl
import oracle
import wl_inputs
from gpu_util import compare

pytestmark = pytest.mark.gpu

# One bf16 rounding of an fp32 sum: |error| <= 2^-8 |W_eff| plus the fp32
# accumulation error of r products (r * 2^-24 * sum |u v|, far below 1e-6 here).
REL = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    wl.lib()


def _ref(p):
    return oracle.theta_reconstruct(p.W0.double().numpy(), p.s.double().numpy(),
                                    p.U.double().numpy(), p.V.double().numpy())


@pytest.mark.parametrize("N,K,r", [(1, 1, 0), (37, 24, 5), (64, 64, 64), (300, 1000, 16),
                                   (129, 130, 65), (513, 72, 256), (100, 200, 1000)])
def test_materialize_elementwise(N, K, r):
    """Tiles of 64 x 64 and rank slices of 64, each with a ragged tail."""
    p = wl_inputs.random_case(400 + N + r, 1, N, K, r).projs[0]
    got = wl.materialize_weight(p.W0.cuda(), p.s.cuda(), p.U.cuda() if r else None,
                                p.V.cuda() if r else None)
    torch.cuda.synchronize()
    ref = _ref(p)
    g = got.double().cpu().numpy()
    bound = REL * np.abs(ref) + 1e-6 * (1 + np.abs(p.U.double().numpy()) @ np.abs(p.V.double().numpy()).T)
    assert np.all(np.abs(g - ref) <= bound), float(np.max(np.abs(g - ref) - bound))


def test_materialize_gemma3_mlp_shape():
    """The Gemma-3-1B gate shape of the decode workloads (4096 x 1152) at rank
    64; 96 rows of W_eff checked in full."""
    p = wl_inputs.random_case(411, 1, 4096, 1152, 64).projs[0]
    got = wl.materialize_weight(p.W0.cuda(), p.s.cuda(), p.U.cuda(), p.V.cuda())
    torch.cuda.synchronize()
    rows = np.random.default_rng(5).choice(4096, 96, replace=False)
    ref = (p.s.double().numpy()[rows, None] * p.W0.double().numpy()[rows]
           + p.U.double().numpy()[rows] @ p.V.double().numpy().T)
    g = got.double().cpu().numpy()[rows]
    assert np.all(np.abs(g - ref) <= REL * np.abs(ref) + 1e-5)


@pytest.mark.parametrize("M", [1, 9, 200])
def test_dense_forward_on_rebuilt_weight(M):
    """x W_eff^T through the rank-0 path equals the theta-bundle forward within
    the forward's tolerance (W_eff carries one extra bf16 rounding)."""
    call = wl_inputs.random_case(420 + M, M, 700, 520, 24)
    p = call.projs[0]
    Weff = wl.materialize_weight(p.W0.cuda(), p.s.cuda(), p.U.cuda(), p.V.cuda())
    ones = torch.ones(700, device="cuda")
    y = wl.linear_forward(call.x.cuda(), Weff, ones, None, None)
    torch.cuda.synchronize()
    assert wl.last_device_status() == 0
    ref = oracle.forward(call.x, p.W0, p.s, p.U, p.V)
    compare(y.double().cpu().numpy(), ref, f"dense M={M}")


def test_materialize_rejects_bad_arguments():
    W0 = torch.ones(4, 8, dtype=torch.bfloat16, device="cuda")
    s = torch.ones(4, device="cuda")
    U = torch.ones(4, 2, dtype=torch.bfloat16, device="cuda")
    with pytest.raises((ValueError, TypeError)):
        wl.materialize_weight(W0, s, U, torch.ones(7, 2, dtype=torch.bfloat16, device="cuda"))
    with pytest.raises((ValueError, TypeError)):
        wl.materialize_weight(W0, s, U, torch.ones(8, 2, dtype=torch.float32, device="cuda"))

"""GPU parity of the NVFP4 decode path (wl_stacked_forward_nvfp4) against the
fp64 NVFP4 oracle (oracle.nvfp4.forward: the dequantised weight, then the
theta-bundle product): ragged row counts, every rank class, stacked calls,
one to eight tokens, a full Gemma-4-31B gate projection, and a weight the
format holds exactly (so the W0 product matches a plain matmul)."""
import numpy as np
import pytest
import torch

import linear_wl_forward_b200 as wl
import wl_inputs
from gpu_util import compare
from oracle import nvfp4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _device():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    wl.lib()


def _case(seed, M, Ns, K, rs):
    projs, host = [], []
    for i, (N, r) in enumerate(zip(Ns, rs)):
        codes, scales, ts = wl_inputs.draw_w0_nvfp4("fp4case", seed, 0, "all", f"f{i}", N, K)
        s, U, V = wl_inputs.draw_delta("fp4case", seed, i, f"f{i}", N, K, r)
        host.append((codes, scales, ts, s, U if r else None, V if r else None))
        projs.append((codes.cuda(), scales.cuda(), ts, s.cuda(), U.cuda() if r else None, V.cuda() if r else None))
    x = wl_inputs.draw_x("fp4case", seed, M, K)
    return x, host, projs


def _check(x, host, projs):
    ys = wl.stacked_forward_nvfp4(x.cuda(), projs)
    torch.cuda.synchronize()
    assert wl.last_device_status() == 0
    for (codes, scales, ts, s, U, V), y in zip(host, ys):
        ref = nvfp4.forward(x, codes.numpy(), scales.numpy(), ts, s, U, V)
        compare(y.double().cpu().numpy(), ref, f"nvfp4 N={codes.shape[0]}")


@pytest.mark.parametrize("M,N,K,r", [(1, 37, 128, 0), (3, 300, 1024, 16), (8, 513, 1152, 64), (5, 1000, 2048, 8),
                                     (2, 129, 384, 256), (1, 16, 4096, 24), (7, 2050, 640, 1024)])
def test_nvfp4_ragged(M, N, K, r):
    _check(*_case(M + N + K + r, M, [N], K, [r]))


@pytest.mark.parametrize("M", [1, 4])
def test_nvfp4_stacked(M):
    _check(*_case(9 + M, M, [300, 64, 1000], 1152, [16, 0, 40]))


def test_nvfp4_gemma4_gate_full_size():
    """A Gemma-4-31B gate projection, 21504 x 5376, rank 256, one token."""
    _check(*_case(4, 1, [21504], 5376, [256]))


def test_nvfp4_exact_weight_equals_matmul():
    """Random codes, unit block scales and a sparse x in {-1, 0, 1}: every
    product and partial sum is a small half-integer (exact in f16 and fp32)
    and so is y, r = 0, s = 1: y equals x W0^T bit for bit."""
    rng = np.random.default_rng(7)
    M, N, K = 3, 48, 256
    nib = rng.integers(0, 16, (N, K)).astype(np.uint8)
    codes = torch.tensor(nib[:, 0::2] | (nib[:, 1::2] << 4))
    scales = torch.full((N, K // 16), 0x38, dtype=torch.uint8)  # E4M3 1.0
    x = torch.tensor(rng.choice([-1, 0, 1], size=(M, K), p=[0.05, 0.9, 0.05]), dtype=torch.bfloat16)
    s = torch.ones(N)
    W0 = nvfp4.dequantize(codes.numpy(), scales.numpy(), 1.0)
    ref = x.double().numpy() @ W0.T
    assert np.array_equal(torch.tensor(ref).to(torch.bfloat16).double().numpy(), ref)
    y = wl.stacked_forward_nvfp4(x.cuda(), [(codes.cuda(), scales.cuda(), 1.0, s.cuda(), None, None)])[0]
    assert np.array_equal(y.double().cpu().numpy(), ref)

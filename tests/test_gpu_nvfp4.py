"""GPU parity of the NVFP4 decode path (wl_stacked_forward_nvfp4) against the
fp64 NVFP4 oracle (oracle.nvfp4.forward: the dequantised weight, then the
theta-bundle product): ragged row counts, every rank class, stacked calls,
one to eight tokens, full Gemma-4-31B gate and down projections, and a weight
the format holds exactly (so the W0 product matches a plain matmul).  Both
weight streams are covered: the persistent ring (K % 256 == 0, K >= 16384,
ranks <= 256, 16-byte-aligned scales, few row blocks per SM), including
blocks split between CTAs, a single block spread over many CTAs and a ragged
last stage, and the one-CTA-per-block stream (the other calls); each case
states which one the plan picks."""
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


def _ring(M, K, projs):
    return wl.describe_nvfp4_plan(M, K, [(p[0].shape[0], 0 if p[4] is None else p[4].shape[1],
                                          p[1].data_ptr() % 16) for p in projs])["ring"]


def _check(x, host, projs, ring=None):
    if ring is not None:
        assert _ring(x.shape[0], x.shape[1], projs) == ring
    ys = wl.stacked_forward_nvfp4(x.cuda(), projs)
    torch.cuda.synchronize()
    assert wl.last_device_status() == 0
    for (codes, scales, ts, s, U, V), y in zip(host, ys):
        ref = nvfp4.forward(x, codes.numpy(), scales.numpy(), ts, s, U, V)
        compare(y.double().cpu().numpy(), ref, f"nvfp4 N={codes.shape[0]}")


@pytest.mark.parametrize("M,N,K,r", [(1, 37, 128, 0), (3, 300, 1024, 16), (8, 513, 1152, 64), (5, 1000, 2048, 8),
                                     (2, 129, 384, 256), (1, 16, 4096, 24), (7, 2050, 640, 1024)])
def test_nvfp4_ragged(M, N, K, r):
    _check(*_case(M + N + K + r, M, [N], K, [r]), ring=0)


@pytest.mark.parametrize("M,N,K,r", [(1, 37, 16384, 0), (3, 300, 16384, 16), (8, 100, 16640, 64),
                                     (2, 513, 16896, 256)])
def test_nvfp4_ring_ragged(M, N, K, r):
    """Ring stream: ragged row counts, and K = 16640 / 16896 whose last
    2048-column stage holds only 2 / 4 of its 16 k-groups."""
    _check(*_case(M + N + K + r, M, [N], K, [r]), ring=1)


@pytest.mark.parametrize("M", [1, 4])
def test_nvfp4_stacked(M):
    _check(*_case(9 + M, M, [300, 64, 1000], 1152, [16, 0, 40]), ring=0)


@pytest.mark.parametrize("M", [1, 3, 8])
def test_nvfp4_ring_stacked_split_blocks(M):
    """Ring stream, three projections (ranks 256, 0, 8) over 148 CTAs: most
    CTA boundaries fall inside a block, whose partial sums the last CTA adds."""
    x, host, projs = _case(30 + M, M, [700, 33, 2000], 16384, [256, 0, 8])
    plan = wl.describe_nvfp4_plan(M, 16384, [(700, 256), (33, 0), (2000, 8)])
    assert plan["ring"] == 1 and plan["grid"] == 148 and plan["units"] % 148 != 0
    _check(x, host, projs, ring=1)


def test_nvfp4_ring_one_block_over_many_ctas():
    """16 rows, K = 21504: one block of 6 stages (4096 columns, the last one
    ragged) and a U unit, one unit per CTA, so 7 CTAs each hold a part of the
    same block."""
    x, host, projs = _case(41, 1, [16], 21504, [256])
    assert wl.describe_nvfp4_plan(1, 21504, [(16, 256)])["grid"] == 7
    _check(x, host, projs, ring=1)


def test_nvfp4_block_stream_when_scales_unaligned_or_rank_large():
    """K >= 16384 with K % 256 == 0 but scales at a 2-byte offset, or a rank
    above 256: the one-CTA-per-block stream."""
    x, host, projs = _case(51, 2, [300, 200], 16384, [16, 512])
    _check(x, host, projs, ring=0)
    x, host, projs = _case(52, 2, [300], 16384, [16])
    codes, scales, ts, s, U, V = projs[0]
    buf = torch.zeros(scales.numel() + 16, dtype=torch.uint8, device="cuda")
    moved = buf[2:2 + scales.numel()].view(scales.shape)
    moved.copy_(scales)
    projs = [(codes, moved, ts, s, U, V)]
    _check(x, host, projs, ring=0)


def test_nvfp4_ring_deterministic():
    x, host, projs = _case(61, 1, [3000, 3000], 16384, [64, 64])
    xd = x.cuda()
    a = [y.clone() for y in wl.stacked_forward_nvfp4(xd, projs)]
    b = wl.stacked_forward_nvfp4(xd, projs)
    torch.cuda.synchronize()
    assert all(torch.equal(p, q) for p, q in zip(a, b))


def test_nvfp4_gemma4_gate_full_size():
    """A Gemma-4-31B gate projection, 21504 x 5376, rank 256, one token (1344
    row blocks: one CTA per block)."""
    _check(*_case(4, 1, [21504], 5376, [256]), ring=0)


def test_nvfp4_gemma4_down_full_size():
    """A Gemma-4-31B down projection, 5376 x 21504, rank 256, two tokens."""
    _check(*_case(5, 2, [5376], 21504, [256]), ring=1)


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

"""Shared helpers of the GPU parity tests: run a Call through the C ABI and
compare with the fp64 oracle under the parity tolerance (max |d| <= 2e-2 max|y_ref|,
relative Frobenius <= 5e-3)."""
import numpy as np
import torch

import linear_wl_forward_b200 as wl
import oracle

# max |delta| <= 2e-2 * max |y_ref| and ||delta||_F / ||y_ref||_F <= 5e-3,
# delta = GPU bf16 output minus the fp64 oracle.
MAX_TOL = 2e-2
FROB_TOL = 5e-3


def to_dev(call):
    x = call.x.cuda()
    projs = [(p.W0.cuda(), p.s.cuda(), p.U.cuda() if p.r else None, p.V.cuda() if p.r else None)
             for p in call.projs]
    return x, projs


def run(call, path="auto", x_dev=None, projs_dev=None):
    x, projs = (x_dev, projs_dev) if x_dev is not None else to_dev(call)
    ys = wl.stacked_forward(x, projs, path=path)
    torch.cuda.synchronize()
    st = wl.last_device_status()
    assert st == 0, f"device status {wl.STATUS.get(st, st)}"
    return [y.float().cpu().numpy().astype(np.float64) for y in ys]


def compare(y_gpu, y_ref, what=""):
    y_ref = np.asarray(y_ref, np.float64)
    if y_ref.size == 0:
        assert y_gpu.size == 0
        return 0.0, 0.0
    d = y_gpu - y_ref
    ref_max = np.max(np.abs(y_ref))
    ref_f = np.linalg.norm(y_ref)
    rel_max = np.max(np.abs(d)) / ref_max if ref_max > 0 else np.max(np.abs(d))
    rel_f = np.linalg.norm(d) / ref_f if ref_f > 0 else np.linalg.norm(d)
    assert np.all(np.isfinite(y_gpu)), what
    assert rel_max <= MAX_TOL, f"{what}: max|d|/max|y| = {rel_max:.3e}"
    assert rel_f <= FROB_TOL, f"{what}: ||d||_F/||y||_F = {rel_f:.3e}"
    return rel_max, rel_f


def check_call(call, path="auto", rows=None):
    """Full check (rows=None) or on the given token rows only."""
    ys = run(call, path)
    x = call.x if rows is None else call.x[rows]
    for p, y in zip(call.projs, ys):
        ref = oracle.forward(x, p.W0, p.s, p.U, p.V)
        compare(y if rows is None else y[rows], ref, f"{p.family} {path} M={call.x.shape[0]}")
    return ys

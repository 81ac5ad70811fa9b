"""Oracle for the theta-bundle linear and its decomposition.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference leg may import this package.  It shares no
code with the CUDA library (``linear_wl_forward_b200``) and never imports it.

* ``forward`` / ``forward_dense``: the plain C fp64 forward (``wl_oracle.c``),
  factored and dense-W_eff forms.
* ``decompose`` / ``relative_frobenius_error``: numpy fp64 decomposition
  (``decompose.py``).
* ``nvfp4``: the NVFP4 weight encoding (E2M1 codes, E4M3 block scales, an
  fp32 tensor scale) and the forward over an NVFP4-encoded W0 (``nvfp4.py``).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from .decompose import (band_of_layer_contiguous, decompose, decompose_als,  # noqa: F401
                        relative_frobenius_error, theta_objective, theta_reconstruct)

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wl_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (plain gcc, fp64, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", _LIB, _SRC])
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        for name in ("wl_oracle_forward", "wl_oracle_forward_dense"):
            fn = getattr(lib, name)
            fn.restype = ctypes.c_int
            fn.argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_long] * 4
        _lib = lib
    return _lib


def _bits(t):
    """bf16 torch tensor (CPU) or uint16 array -> contiguous uint16 numpy array."""
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch

    assert t.dtype == torch.bfloat16, t.dtype
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _f32(t):
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float32)
    return t.detach().cpu().contiguous().numpy().astype(np.float32, copy=False)


def _run(name, x, W0, s, U, V, lib=None):
    """Marshal the operands and call `name` in the oracle library (or in
    `lib`, a library built from a modified copy of the same source)."""
    lib = _load() if lib is None else lib
    xb, wb, sb = _bits(x), _bits(W0), _f32(s)
    M, K = xb.shape
    N = wb.shape[0]
    assert wb.shape == (N, K) and sb.shape == (N,)
    if U is None or (hasattr(U, "shape") and U.shape[-1] == 0):
        r = 0
        ub = np.zeros((N, 0), np.uint16)
        vb = np.zeros((K, 0), np.uint16)
    else:
        ub, vb = _bits(U), _bits(V)
        r = ub.shape[1]
        assert ub.shape == (N, r) and vb.shape == (K, r)
    y = np.empty((M, N), np.float64)
    rc = getattr(lib, name)(xb.ctypes.data, wb.ctypes.data, sb.ctypes.data,
                            ub.ctypes.data, vb.ctypes.data, y.ctypes.data, M, N, K, r)
    if rc != 0:
        raise MemoryError(name)
    return y


def forward(x, W0, s, U, V):
    """y = s * (W0 x) + U (V^T x) in fp64 (factored steps).  x: M x K bf16,
    W0: N x K bf16, s: N fp32, U: N x r bf16, V: K x r bf16 -> y: M x N fp64."""
    return _run("wl_oracle_forward", x, W0, s, U, V)


def forward_dense(x, W0, s, U, V):
    """y = (diag(s) W0 + U V^T) x in fp64 (dense effective weight)."""
    return _run("wl_oracle_forward_dense", x, W0, s, U, V)

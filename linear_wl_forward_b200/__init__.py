"""Python binding of the B200 theta-bundle linear (``libwl.so``, include/wl.h).

Argument marshalling only: torch tensors are checked for dtype, device and
layout and their pointers are handed to the C ABI; every step of the forward
runs in the library's CUDA kernels.  There is no fallback: if the library is
missing or was built for another device, calls raise.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "WLError", "lib", "linear_forward", "stacked_forward", "prepare_stacked", "PreparedForward",
    "prefetch_ranges", "MAX_PREFETCH", "stacked_forward_nvfp4", "NVFP4_MAX_M",
    "materialize_weight", "describe_decode_plan", "DecodePlan", "describe_rows_plan", "RowsPlan",
    "describe_nvfp4_plan", "Nvfp4Plan",
    "quantize_nvfp4",
    "decompose",
    "relative_frobenius_error", "last_device_status", "wait_probe", "set_wait_limit", "PATHS",
    "DECODE_MAX_M", "MAX_RANK", "MAX_PROJ", "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwl.so")

STATUS = {0: "WL_OK", 1: "WL_ERR_INVALID_ARG", 2: "WL_ERR_ALIGNMENT", 3: "WL_ERR_UNSUPPORTED",
          4: "WL_ERR_CUDA", 5: "WL_ERR_TIMEOUT", 6: "WL_ERR_NOMEM", 7: "WL_ERR_NOT_CONVERGED"}
PATHS = {"auto": 0, "decode": 1, "gemm": 2, "rows": 3, "ring": 4}
DECODE_MAX_M = 16
MAX_RANK = 1024
MAX_PROJ = 8
MAX_PREFETCH = 32
NVFP4_MAX_M = 8


class WLError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        self.name = STATUS.get(code, str(code))
        super().__init__(f"{what}: {self.name} ({_lib.wl_status_string(code).decode() if _lib else ''})")


class _Proj(ctypes.Structure):
    _fields_ = [("W0", ctypes.c_void_p), ("s", ctypes.c_void_p), ("U", ctypes.c_void_p),
                ("V", ctypes.c_void_p), ("y", ctypes.c_void_p), ("N", ctypes.c_int),
                ("r", ctypes.c_int)]


class _Range(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("bytes", ctypes.c_size_t)]


class _ProjNvfp4(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("tensor_scale", ctypes.c_float),
                ("s", ctypes.c_void_p), ("U", ctypes.c_void_p), ("V", ctypes.c_void_p), ("y", ctypes.c_void_p),
                ("N", ctypes.c_int), ("r", ctypes.c_int)]


class RowsPlan(ctypes.Structure):
    """wl_rows_plan of include/wl.h."""
    _fields_ = [("grid", ctypes.c_int), ("cluster", ctypes.c_int), ("row_groups", ctypes.c_int),
                ("nb_max", ctypes.c_int), ("k_slice", ctypes.c_int), ("smem_bytes", ctypes.c_longlong)]


class Nvfp4Plan(ctypes.Structure):
    """wl_nvfp4_plan of include/wl.h."""
    _fields_ = [("ring", ctypes.c_int), ("grid", ctypes.c_int), ("stages", ctypes.c_int),
                ("slot_bytes", ctypes.c_int), ("smem_bytes", ctypes.c_int), ("units", ctypes.c_longlong),
                ("prep_slices", ctypes.c_int), ("prep_rows", ctypes.c_int), ("prep_grid", ctypes.c_int)]


class DecodePlan(ctypes.Structure):
    """wl_decode_plan of include/wl.h."""
    _fields_ = [("auto_decode", ctypes.c_int), ("grid", ctypes.c_int), ("compact", ctypes.c_int),
                ("smem_bytes", ctypes.c_longlong), ("t_mode", ctypes.c_int), ("t_fused", ctypes.c_int),
                ("seg_split", ctypes.c_int), ("slots", ctypes.c_int), ("slot_chunks", ctypes.c_int),
                ("x_smem", ctypes.c_int), ("v_stage", ctypes.c_int), ("v_in_ring", ctypes.c_int),
                ("u_stage", ctypes.c_int), ("lag", ctypes.c_int)]


_lib = None


def lib():
    """Loads libwl.so (built by ``python -m linear_wl_forward_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m linear_wl_forward_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, ci, cll = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
        L.wl_linear_forward.argtypes = [vp] * 6 + [ci] * 4 + [vp]
        L.wl_stacked_forward.argtypes = [vp, ci, ci, ctypes.POINTER(_Proj), ci, vp]
        L.wl_forward_ex.argtypes = [vp, ci, ci, ctypes.POINTER(_Proj), ci, ci, vp]
        L.wl_stacked_forward_prefetch.argtypes = [vp, ci, ci, ctypes.POINTER(_Proj), ci, ci,
                                                  ctypes.POINTER(_Range), ci, vp]
        L.wl_decompose.argtypes = [vp, ci, ci, ci, ci, ci, vp, vp, vp, vp, vp, vp]
        L.wl_decompose_als.argtypes = [vp, ci, ci, ci, ci, ci, vp, ci, vp, vp, vp, vp, vp]
        L.wl_materialize_weight.argtypes = [vp, vp, vp, vp, vp, ci, ci, ci, vp]
        L.wl_describe_decode_plan.argtypes = [ci, ci, ctypes.POINTER(_Proj), ci, ci,
                                              ctypes.POINTER(DecodePlan)]
        L.wl_stacked_forward_nvfp4.argtypes = [vp, ci, ci, ctypes.POINTER(_ProjNvfp4), ci, vp]
        L.wl_describe_rows_plan.argtypes = [ci, ci, ctypes.POINTER(_Proj), ci, ci, ctypes.POINTER(RowsPlan)]
        L.wl_describe_nvfp4_plan.argtypes = [ci, ci, ctypes.POINTER(_ProjNvfp4), ci, ci, ctypes.POINTER(Nvfp4Plan)]
        L.wl_quantize_nvfp4.argtypes = [vp, ci, ci, ctypes.c_float, vp, vp, ctypes.POINTER(ctypes.c_float)]
        L.wl_relative_frobenius_error.argtypes = [vp] * 5 + [ci] * 3
        L.wl_relative_frobenius_error.restype = ctypes.c_double
        L.wl_status_string.argtypes = [ci]
        L.wl_status_string.restype = ctypes.c_char_p
        L.wl_last_device_status.argtypes = [vp]
        L.wl_wait_probe.argtypes = [cll, vp]
        L.wl_set_wait_limit.argtypes = [cll]
        L.wl_noalloc_last_status.argtypes = [vp]
        L.wl_version.restype = ci
        for name in ("wl_linear_forward", "wl_stacked_forward", "wl_forward_ex", "wl_stacked_forward_prefetch",
                     "wl_stacked_forward_nvfp4",
                     "wl_decompose", "wl_decompose_als",
                     "wl_materialize_weight", "wl_describe_decode_plan", "wl_describe_rows_plan",
                     "wl_describe_nvfp4_plan",
                     "wl_quantize_nvfp4",
                     "wl_last_device_status", "wl_wait_probe", "wl_set_wait_limit", "wl_noalloc_last_status"):
            getattr(L, name).restype = ci
        _lib = L
    return _lib


def _check(code: int, what: str):
    if code != 0:
        raise WLError(code, what)


def _stream_handle(stream):
    import torch

    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dev_ptr(t, dtype, name, shape=None):
    import torch

    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return t.data_ptr()


def _make_proj(W0, s, U, V, y, M, K):
    import torch

    N = W0.shape[0]
    r = 0 if U is None else U.shape[1]
    return _Proj(_dev_ptr(W0, torch.bfloat16, "W0", (N, K)), _dev_ptr(s, torch.float32, "s", (N,)),
                 _dev_ptr(U, torch.bfloat16, "U", (N, r)) if r else None,
                 _dev_ptr(V, torch.bfloat16, "V", (K, r)) if r else None,
                 _dev_ptr(y, torch.bfloat16, "y", (M, N)), N, r)


def linear_forward(x, W0, s, U, V, y=None, stream=None, path="auto"):
    """y = s * (W0 x) + U (V^T x).  x: M x K bf16, W0: N x K bf16, s: N fp32,
    U: N x r bf16, V: K x r bf16 (U = V = None for r = 0).  Returns y (M x N
    bf16); asynchronous on `stream` (default: torch's current stream)."""
    return stacked_forward(x, [(W0, s, U, V)], ys=None if y is None else [y], stream=stream,
                           path=path)[0]


def stacked_forward_nvfp4(x, projs, ys=None, stream=None):
    """The stacked forward with NVFP4 shared blocks (include/wl.h,
    wl_stacked_forward_nvfp4).  projs: (codes N x K/2 uint8, scales N x K/16
    uint8, tensor_scale float, s, U, V) per projection, CUDA tensors (U = V =
    None for r = 0).  Returns the list of y_p (M x N_p bf16)."""
    import torch

    M, K = x.shape
    if ys is None:
        ys = [torch.empty(M, c.shape[0], dtype=torch.bfloat16, device=x.device) for (c, *_rest) in projs]
    arr = (_ProjNvfp4 * len(projs))()
    for i, ((codes, scales, ts, s, U, V), y) in enumerate(zip(projs, ys)):
        N = codes.shape[0]
        r = 0 if U is None else U.shape[1]
        arr[i] = _ProjNvfp4(_dev_ptr(codes, torch.uint8, "codes", (N, K // 2)),
                            _dev_ptr(scales, torch.uint8, "scales", (N, K // 16)), float(ts),
                            _dev_ptr(s, torch.float32, "s", (N,)),
                            _dev_ptr(U, torch.bfloat16, "U", (N, r)) if r else None,
                            _dev_ptr(V, torch.bfloat16, "V", (K, r)) if r else None,
                            _dev_ptr(y, torch.bfloat16, "y", (M, N)), N, r)
    _check(lib().wl_stacked_forward_nvfp4(_dev_ptr(x, torch.bfloat16, "x", (M, K)), M, K, arr, len(projs),
                                          _stream_handle(stream)), "wl_stacked_forward_nvfp4")
    return ys


def prefetch_ranges(items):
    """wl_range array for wl_stacked_forward_prefetch from CUDA tensors (their
    whole storage from data_ptr) and/or (device address, bytes) pairs; None
    entries are skipped."""
    import torch

    ranges = []
    for it in items:
        if it is None:
            continue
        if isinstance(it, torch.Tensor):
            if not it.is_cuda:
                raise TypeError("prefetch tensors must be CUDA tensors")
            ranges.append((it.data_ptr(), it.numel() * it.element_size()))
        else:
            ptr, nbytes = it
            ranges.append((int(ptr), int(nbytes)))
    if len(ranges) > MAX_PREFETCH:
        raise ValueError(f"at most {MAX_PREFETCH} prefetch ranges, got {len(ranges)}")
    return (_Range * max(len(ranges), 1))(*[_Range(p, n) for p, n in ranges]), len(ranges)


def stacked_forward(x, projs, ys=None, stream=None, path="auto", prefetch=None):
    """Several projections (W0_p, s_p, U_p, V_p) against one shared x in one
    call.  Returns the list of y_p (M x N_p bf16).  `prefetch`: tensors (or
    (address, bytes) pairs) to pull into L2 while the call runs, normally the
    weights of the call that follows (include/wl.h, wl_stacked_forward_prefetch)."""
    import torch

    M, K = x.shape
    if ys is None:
        ys = [torch.empty(M, W0.shape[0], dtype=torch.bfloat16, device=x.device)
              for (W0, _, _, _) in projs]
    arr = (_Proj * len(projs))(*[_make_proj(W0, s, U, V, y, M, K)
                                 for (W0, s, U, V), y in zip(projs, ys)])
    xp = _dev_ptr(x, torch.bfloat16, "x", (M, K))
    if prefetch:
        rng, n = prefetch_ranges(prefetch)
        _check(lib().wl_stacked_forward_prefetch(xp, M, K, arr, len(projs), PATHS[path], rng, n,
                                                 _stream_handle(stream)), "wl_stacked_forward_prefetch")
    else:
        _check(lib().wl_forward_ex(xp, M, K, arr, len(projs), PATHS[path], _stream_handle(stream)),
               "wl_forward_ex")
    return ys


class PreparedForward:
    """A stacked forward whose tensors are checked and marshalled once.

    Calling it issues the forward on `stream` (default: torch's current
    stream) with the same tensors; it returns the list of y_p.  A decode step
    that runs the same projections on the same buffers every token calls
    these instead of ``stacked_forward`` and so pays the checks once.  The
    tensors are kept alive by this object; their storage must not be
    replaced (in-place writes to x and the weights between calls are fine).
    """

    def __init__(self, x, projs, ys=None, path="auto", prefetch=None):
        import torch

        M, K = x.shape
        if ys is None:
            ys = [torch.empty(M, W0.shape[0], dtype=torch.bfloat16, device=x.device)
                  for (W0, _, _, _) in projs]
        self.ys = ys
        self._keep = (x, projs, ys, prefetch)
        self._arr = (_Proj * len(projs))(*[_make_proj(W0, s, U, V, y, M, K)
                                           for (W0, s, U, V), y in zip(projs, ys)])
        self._rng, self._nrng = prefetch_ranges(prefetch or [])
        self._args = (_dev_ptr(x, torch.bfloat16, "x", (M, K)), M, K, self._arr, len(projs), PATHS[path])
        self._fn = lib().wl_stacked_forward_prefetch

    def __call__(self, stream=None):
        xp, M, K, arr, P, path = self._args
        _check(self._fn(xp, M, K, arr, P, path, self._rng, self._nrng, _stream_handle(stream)),
               "wl_stacked_forward_prefetch")
        return self.ys


def prepare_stacked(x, projs, ys=None, path="auto", prefetch=None) -> PreparedForward:
    """``stacked_forward`` with its argument checks done once: returns a
    callable that issues the forward (see PreparedForward).  `prefetch` as in
    ``stacked_forward``."""
    return PreparedForward(x, projs, ys, path, prefetch)


def materialize_weight(W0, s, U, V, out=None, stream=None):
    """W_eff = diag(s) W0 + U V^T (N x K bf16) on the GPU: the dense weight the
    bundle stands for, for the precompute-outside path (a dense forward is
    then ``linear_forward(x, W_eff, ones, None, None)``)."""
    import torch

    N, K = W0.shape
    r = 0 if U is None else U.shape[1]
    if out is None:
        out = torch.empty(N, K, dtype=torch.bfloat16, device=W0.device)
    _check(lib().wl_materialize_weight(
        _dev_ptr(W0, torch.bfloat16, "W0", (N, K)), _dev_ptr(s, torch.float32, "s", (N,)),
        _dev_ptr(U, torch.bfloat16, "U", (N, r)) if r else None,
        _dev_ptr(V, torch.bfloat16, "V", (K, r)) if r else None,
        _dev_ptr(out, torch.bfloat16, "out", (N, K)), N, K, r, _stream_handle(stream)),
        "wl_materialize_weight")
    return out


def quantize_nvfp4(W, tensor_scale: float = 0.0):
    """NVFP4 encoding on the host (include/wl.h, wl_quantize_nvfp4).  W: N x K
    float32 numpy array, K % 16 == 0.  Returns (codes N x K/2 uint8, scales
    N x K/16 uint8, tensor scale); tensor_scale 0 derives it from max|W|."""
    import numpy as np

    W = np.ascontiguousarray(W, dtype=np.float32)
    N, K = W.shape
    codes = np.empty((N, K // 2), np.uint8)
    scales = np.empty((N, max(K // 16, 0)), np.uint8)
    ts = ctypes.c_float(0.0)
    _check(lib().wl_quantize_nvfp4(W.ctypes.data, N, K, float(tensor_scale), codes.ctypes.data,
                                   scales.ctypes.data, ctypes.byref(ts)), "wl_quantize_nvfp4")
    return codes, scales, ts.value


def describe_decode_plan(M: int, K: int, projs, num_sms: int = 148) -> dict:
    """The decode kernel's host-side plan for a call, made without a GPU.

    ``projs`` holds ``(N, r)`` pairs, or ``(N, r, uv_offset)`` with U and V
    placed ``uv_offset`` bytes past a 16-byte boundary.  The pointers handed
    to the library are stand-ins: it checks them for NULL and alignment only.
    Raises WLError for shapes the decode kernel declines."""
    arr = (_Proj * len(projs))()
    for i, q in enumerate(projs):
        N, r = q[0], q[1]
        off = q[2] if len(q) > 2 else 0
        base = (i + 1) << 32
        arr[i] = _Proj(base, base + (1 << 28), (base + (2 << 28) + off) if r else None,
                       (base + (3 << 28) + off) if r else None, base + (4 << 28), N, r)
    out = DecodePlan()
    _check(lib().wl_describe_decode_plan(M, K, arr, len(projs), num_sms, ctypes.byref(out)),
           "wl_describe_decode_plan")
    return {name: getattr(out, name) for name, _ in DecodePlan._fields_}


def _stand_in_projs(projs):
    arr = (_Proj * len(projs))()
    for i, q in enumerate(projs):
        N, r = q[0], q[1]
        off = q[2] if len(q) > 2 else 0
        base = (i + 1) << 32
        arr[i] = _Proj(base, base + (1 << 28), (base + (2 << 28) + off) if r else None,
                       (base + (3 << 28) + off) if r else None, base + (4 << 28), N, r)
    return arr


def describe_rows_plan(M: int, K: int, projs, num_sms: int = 148) -> dict:
    """The row-stream kernel's host-side plan for a call, made without a GPU
    (``projs`` as in ``describe_decode_plan``).  Raises WLError (code 3) for
    calls the kernel does not take."""
    arr = _stand_in_projs(projs)
    out = RowsPlan()
    _check(lib().wl_describe_rows_plan(M, K, arr, len(projs), num_sms, ctypes.byref(out)),
           "wl_describe_rows_plan")
    return {name: getattr(out, name) for name, _ in RowsPlan._fields_}


def describe_nvfp4_plan(M: int, K: int, projs, num_sms: int = 148) -> dict:
    """The NVFP4 forward's host-side plan for a call, made without a GPU.
    ``projs``: (N, r) or (N, r, scales_offset_bytes) per projection; stand-in
    addresses (never dereferenced) are 16-byte aligned, the scales moved by
    the offset."""
    arr = (_ProjNvfp4 * len(projs))()
    for i, q in enumerate(projs):
        N, r = q[0], q[1]
        off = q[2] if len(q) > 2 else 0
        base = (i + 1) << 32
        arr[i] = _ProjNvfp4(base, base + (1 << 28) + off, 1.0, base + (2 << 28),
                            (base + (3 << 28)) if r else None, (base + (4 << 28)) if r else None,
                            base + (5 << 28), N, r)
    out = Nvfp4Plan()
    _check(lib().wl_describe_nvfp4_plan(M, K, arr, len(projs), num_sms, ctypes.byref(out)),
           "wl_describe_nvfp4_plan")
    return {name: getattr(out, name) for name, _ in Nvfp4Plan._fields_}


def last_device_status(stream=None) -> int:
    """Synchronises the stream and returns (and clears) the device status word."""
    return lib().wl_last_device_status(_stream_handle(stream))


def set_wait_limit(limit_ns: int):
    """Time limit of the device-side waits of later forward calls (0: the
    default, 2 s); for tests of the time-out path."""
    _check(lib().wl_set_wait_limit(int(limit_ns)), "wl_set_wait_limit")


def wait_probe(limit_ns: int, stream=None):
    _check(lib().wl_wait_probe(int(limit_ns), _stream_handle(stream)), "wl_wait_probe")


def decompose(W, G: int, r: int, band_of_layer=None, als_iters: int = 0):
    """Host decomposition (include/wl.h, wl_decompose; with als_iters > 0,
    wl_decompose_als: that many alternating-least-squares rounds over the
    band-mean start).  W: (L, N, K) float32 numpy array.  Returns
    (W0 (G,N,K), s (L,N), U (L,N,r), V (L,K,r), rel_err (L,))."""
    import numpy as np

    W = np.ascontiguousarray(W, dtype=np.float32)
    L, N, K = W.shape
    W0 = np.empty((G, N, K), np.float32)
    s = np.empty((L, N), np.float32)
    U = np.empty((L, N, r), np.float32)
    V = np.empty((L, K, r), np.float32)
    err = np.empty(L, np.float64)
    bands = None
    if band_of_layer is not None:
        bands = np.ascontiguousarray(band_of_layer, dtype=np.int32)
    bp = None if bands is None else bands.ctypes.data
    if als_iters:
        _check(lib().wl_decompose_als(W.ctypes.data, L, N, K, G, r, bp, int(als_iters), W0.ctypes.data,
                                      s.ctypes.data, U.ctypes.data, V.ctypes.data, err.ctypes.data),
               "wl_decompose_als")
    else:
        _check(lib().wl_decompose(W.ctypes.data, L, N, K, G, r, bp, W0.ctypes.data,
                                  s.ctypes.data, U.ctypes.data, V.ctypes.data, err.ctypes.data),
               "wl_decompose")
    return W0, s, U, V, err


def relative_frobenius_error(W, W0, s, U, V) -> float:
    import numpy as np

    W, W0, s = (np.ascontiguousarray(a, dtype=np.float32) for a in (W, W0, s))
    N, K = W.shape
    r = 0 if U is None else U.shape[1]
    U = np.ascontiguousarray(U, dtype=np.float32) if r else None
    V = np.ascontiguousarray(V, dtype=np.float32) if r else None
    return lib().wl_relative_frobenius_error(W.ctypes.data, W0.ctypes.data, s.ctypes.data,
                                             None if U is None else U.ctypes.data,
                                             None if V is None else V.ctypes.data, N, K, r)

"""C-ABI checks that need no GPU: the library loads, exports every function
include/wl.h declares, and rejects bad arguments on the host before touching
CUDA."""
import ctypes
import os
import re

import pytest

import linear_wl_forward_b200 as wl
from linear_wl_forward_b200 import build as wlbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    wlbuild.build()
    return wl.lib()


def header_functions():
    text = open(os.path.join(ROOT, "include", "wl.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(wl_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_function(L):
    names = header_functions()
    assert "wl_linear_forward" in names and "wl_decompose" in names
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for code in range(8):
        assert L.wl_status_string(code)
    assert b"converge" in L.wl_status_string(7)
    assert L.wl_version() >= 1


FAKE = 0x10000  # 16-byte aligned fake device address; never dereferenced


def call(L, x=FAKE, W0=FAKE, s=FAKE, U=FAKE, V=FAKE, y=FAKE, M=1, N=8, K=16, r=8):
    return L.wl_linear_forward(x, W0, s, U, V, y, M, N, K, r, None)


def test_host_validation(L):
    assert call(L, x=None) == 1                  # null x
    assert call(L, W0=None) == 1
    assert call(L, s=None) == 1
    assert call(L, y=None) == 1
    assert call(L, U=None) == 1                  # r > 0 needs U and V
    assert call(L, M=-1) == 1
    assert call(L, N=-2) == 1
    assert call(L, r=-1) == 1
    assert call(L, K=12) == 2                    # K % 8 != 0
    assert call(L, x=FAKE + 2) == 2              # misaligned x
    assert call(L, W0=FAKE + 8) == 2             # misaligned W0
    assert call(L, r=wl.MAX_RANK + 1) == 3
    # empty inputs are a no-op and touch nothing
    assert call(L, M=0, x=None, y=None) == 0
    assert call(L, N=0, W0=None, s=None, y=None, U=None, V=None) == 0


def test_stacked_validation(L):
    P = wl.MAX_PROJ + 1
    arr = (wl._Proj * P)(*[wl._Proj(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 8) for _ in range(P)])
    assert L.wl_stacked_forward(FAKE, 1, 16, arr, P, None) == 3
    assert L.wl_stacked_forward(FAKE, 1, 16, arr, 0, None) == 1
    assert L.wl_stacked_forward(FAKE, 1, 16, None, 1, None) == 1
    # the decode path serves at most WL_DECODE_MAX_M tokens
    assert L.wl_forward_ex(FAKE, wl.DECODE_MAX_M + 1, 16, arr, 1, wl.PATHS["decode"], None) == 3
    assert L.wl_forward_ex(FAKE, 1, 16, arr, 1, 7, None) == 1


def test_wait_probe_rejects_bad_limit(L):
    assert L.wl_wait_probe(0, None) == 1
    assert L.wl_wait_probe(2_000_000_000, None) == 1


def test_materialize_validation(L):
    def mat(W0=FAKE, s=FAKE, U=FAKE, V=FAKE, out=FAKE, N=8, K=16, r=4):
        return L.wl_materialize_weight(W0, s, U, V, out, N, K, r, None)

    assert mat(N=-1) == 1
    assert mat(K=-1) == 1
    assert mat(r=-1) == 1
    assert mat(r=wl.MAX_RANK + 1) == 3
    assert mat(W0=None) == 1
    assert mat(s=None) == 1
    assert mat(out=None) == 1
    assert mat(U=None) == 1                  # r > 0 needs U and V
    assert mat(V=None) == 1
    # empty weights are a no-op and touch nothing
    assert mat(N=0, W0=None, s=None, U=None, V=None, out=None) == 0
    assert mat(K=0, W0=None, s=None, U=None, V=None, out=None) == 0


def test_prefetch_validation(L):
    """wl_stacked_forward_prefetch rejects bad range lists on the host, before
    anything is launched."""
    arr = (wl._Proj * 1)(wl._Proj(FAKE, FAKE, FAKE, FAKE, FAKE, 8, 8))
    rng = (wl._Range * (wl.MAX_PREFETCH + 1))()
    fn = L.wl_stacked_forward_prefetch
    assert fn(FAKE, 1, 16, arr, 1, 0, rng, -1, None) == 1
    assert fn(FAKE, 1, 16, arr, 1, 0, rng, wl.MAX_PREFETCH + 1, None) == 1
    assert fn(FAKE, 1, 16, arr, 1, 0, None, 1, None) == 1
    rng[0] = wl._Range(None, 64)  # a NULL range with bytes
    assert fn(FAKE, 1, 16, arr, 1, 0, rng, 1, None) == 1
    # the call's own checks come first
    assert fn(FAKE, 1, 12, arr, 1, 0, rng, 0, None) == 2
    # empty calls are a no-op whatever the list holds
    assert fn(FAKE, 0, 16, arr, 1, 0, rng, 0, None) == 0


def test_wait_limit_validation(L):
    assert L.wl_set_wait_limit(-1) == 1
    assert L.wl_set_wait_limit(20_000_000_000) == 1
    assert L.wl_set_wait_limit(1000) == 0
    assert L.wl_set_wait_limit(0) == 0  # back to the default


def test_nvfp4_validation(L):
    """wl_stacked_forward_nvfp4 rejects bad calls on the host."""
    def call(M=1, K=128, N=16, r=8, ts=0.5, codes=FAKE, scales=FAKE, U=FAKE, V=FAKE):
        arr = (wl._ProjNvfp4 * 1)(wl._ProjNvfp4(codes, scales, ts, FAKE, U, V, FAKE, N, r))
        return L.wl_stacked_forward_nvfp4(FAKE, M, K, arr, 1, None)

    assert call(K=64) == 2                 # K % 128
    assert call(codes=FAKE + 8) == 2       # codes 16-byte aligned
    assert call(scales=FAKE + 1) == 2      # scales 2-byte aligned
    assert call(r=12) == 2                 # rank % 8
    assert call(U=FAKE + 8) == 2           # U 16-byte aligned
    assert call(V=FAKE + 8) == 2           # V 16-byte aligned
    assert call(ts=0.0) == 1
    assert call(ts=-1.0) == 1
    assert call(ts=float("inf")) == 1
    assert call(M=wl.NVFP4_MAX_M + 1) == 3
    assert call(r=wl.MAX_RANK + 8) == 3
    assert call(M=0) == 0                  # empty calls touch nothing
    assert L.wl_stacked_forward_nvfp4(FAKE, 1, 128, None, 1, None) == 1


def test_nvfp4_plan_picks_the_stream():
    """wl_describe_nvfp4_plan: the ring stream for K % 256 == 0, ranks <= 256,
    16-byte-aligned scales and K >= 8192 or at least 2048 row blocks; one CTA
    per 16-row block otherwise.  The ring's shared memory fits a CTA and its
    units cover the call."""
    ring = wl.describe_nvfp4_plan(1, 21504, [(5376, 256)])      # Gemma-4 down
    assert ring["ring"] == 1 and ring["grid"] == 148
    assert ring["units"] == 336 * (6 + 1)            # 336 blocks x (6 stages of 4096 columns + U) each
    assert ring["smem_bytes"] <= 227 * 1024 and ring["stages"] >= 2
    assert ring["prep_grid"] == ring["prep_slices"]
    assert ring["prep_slices"] * ring["prep_rows"] >= 21504
    gate_up = wl.describe_nvfp4_plan(1, 5376, [(21504, 256), (21504, 256)])
    assert gate_up["ring"] == 1 and gate_up["grid"] == 148           # 2688 blocks
    assert gate_up["prep_grid"] == 2 * gate_up["prep_slices"]
    q = wl.describe_nvfp4_plan(1, 5376, [(8192, 256)])
    assert q["ring"] == 0 and q["grid"] == 8192 // 16                 # 512 blocks over a short K
    assert wl.describe_nvfp4_plan(1, 8192, [(5376, 256)])["ring"] == 1       # Gemma-4 o: K = 8192
    for M in range(1, wl.NVFP4_MAX_M + 1):
        p = wl.describe_nvfp4_plan(M, 16384, [(700, 256)])
        assert p["ring"] == 1 and p["smem_bytes"] <= 227 * 1024 and p["stages"] >= 2
    assert wl.describe_nvfp4_plan(1, 1152, [(300, 16)])["ring"] == 0          # K % 256 != 0
    assert wl.describe_nvfp4_plan(1, 16384, [(300, 512)])["ring"] == 0        # rank > 256
    assert wl.describe_nvfp4_plan(1, 16384, [(300, 16, 2)])["ring"] == 0      # scales at +2 bytes
    assert wl.describe_nvfp4_plan(1, 16384, [(300, 16)])["ring"] == 1
    blocks = wl.describe_nvfp4_plan(1, 1152, [(300, 16)])
    assert blocks["grid"] == (300 + 15) // 16
    tiny = wl.describe_nvfp4_plan(1, 16384, [(16, 24)])
    assert tiny["ring"] == 1 and tiny["grid"] == tiny["units"] == 4 + 1   # 4 stages of 4096 columns + U

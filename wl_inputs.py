"""Seeded synthetic inputs for the theta-bundle linear (shared by the tests, the
bench and the oracle checks).

This module holds workload SHAPES and random draws only.  It contains none of
the method's arithmetic: no forward, no decomposition, no scaling.

Every tensor is drawn on the CPU from its own ``torch.Generator`` whose seed is
a stable hash of (workload, seed, scope, family, tensor name), drawn in fp32
and then rounded to the storage type (RNE to bf16 where the bundle is bf16).

Distributions (the synthetic stand-ins for the Gemma checkpoints, which are not
available): W0, U, V ~ N(0, 0.02) bf16; s ~ U(0.9, 1.1) fp32; x ~ N(0, 1) bf16.

Shapes follow the Gemma 3 1B and Gemma 4 31B projection families described on
the "Quality (Gemma 4 31B)" page (architecture and weight shapes) and the
"Compression" page (theta-bundle size, Gemma 3 1B dimensions: 26 layers,
hidden 1152, intermediate 4096).
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass, field

import torch

W_STD = 0.02
S_LO, S_HI = 0.9, 1.1

# ---------------------------------------------------------------- shapes ----
# (N, K) per projection family: N output rows, K inputs (Linear.weight layout).
GEMMA3_1B_FAMILIES = {
    "q": (1024, 1152),
    "k": (256, 1152),
    "v": (256, 1152),
    "o": (1152, 1024),
    "gate": (4096, 1152),
    "up": (4096, 1152),
    "down": (1152, 4096),
}
GEMMA3_1B_LAYERS = 26
GEMMA3_1B_STACKS = [("q", "k", "v"), ("o",), ("gate", "up"), ("down",)]

GEMMA4_31B_SLIDING = {
    "q": (8192, 5376),
    "k": (4096, 5376),
    "v": (4096, 5376),
    "o": (5376, 8192),
}
GEMMA4_31B_FULL = {
    "q": (16384, 5376),
    "k": (2048, 5376),  # k = v tied on full-attention layers: no v projection
    "o": (5376, 16384),
}
GEMMA4_31B_MLP = {
    "gate": (21504, 5376),
    "up": (21504, 5376),
    "down": (5376, 21504),
}
GEMMA4_31B_LAYERS = 60
GEMMA4_31B_BANDS = 5


def gemma4_layer_type(layer: int) -> str:
    """10 full-attention + 50 sliding layers; full iff layer % 6 == 5 (a reading:
    the pages give the counts, not the pattern)."""
    return "full" if layer % 6 == 5 else "sliding"


def gemma4_families(layer_type: str) -> dict:
    fam = dict(GEMMA4_31B_SLIDING if layer_type == "sliding" else GEMMA4_31B_FULL)
    fam.update(GEMMA4_31B_MLP)
    return fam


def gemma4_stacks(layer_type: str):
    if layer_type == "sliding":
        return [("q", "k", "v"), ("o",), ("gate", "up"), ("down",)]
    return [("q", "k"), ("o",), ("gate", "up"), ("down",)]


def contiguous_band(layer: int, num_layers: int, num_bands: int) -> int:
    """Contiguous equal bands: band(l) = floor(l * G / L)."""
    return (layer * num_bands) // num_layers


# ------------------------------------------------------------- seeding ------
def subseed(*key) -> int:
    h = hashlib.sha256("|".join(str(k) for k in key).encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(*key) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(subseed(*key))
    return g


def normal_bf16(shape, std, *key) -> torch.Tensor:
    t = torch.randn(*shape, generator=_gen(*key), dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(torch.bfloat16)


def uniform_f32(shape, lo, hi, *key) -> torch.Tensor:
    t = torch.rand(*shape, generator=_gen(*key), dtype=torch.float32)
    return t.mul_(hi - lo).add_(lo)


def draw_w0(workload: str, seed: int, band: int, layer_type: str, family: str,
            N: int, K: int) -> torch.Tensor:
    return normal_bf16((N, K), W_STD, workload, seed, "W0", band, layer_type, family)


def draw_delta(workload: str, seed: int, layer: int, family: str, N: int, K: int,
               r: int):
    """Per-layer (s, U, V): s fp32[N], U bf16[N, r], V bf16[K, r]."""
    s = uniform_f32((N,), S_LO, S_HI, workload, seed, "s", layer, family)
    U = normal_bf16((N, r), W_STD, workload, seed, "U", layer, family)
    V = normal_bf16((K, r), W_STD, workload, seed, "V", layer, family)
    return s, U, V


# NVFP4-encoded W0, drawn directly as bytes (no encoding arithmetic here): the
# magnitude code of each element follows roughly the mix a block-scaled
# Gaussian row gives (most elements small, few at the block maximum), the sign
# is even, and the block scale bytes are E4M3 codes 0x30..0x4F (0.5 .. 15),
# around a tensor scale of 2^-9, so dequantised weights are of order 0.01.
NVFP4_MAG_WEIGHTS = (0.10, 0.18, 0.17, 0.14, 0.17, 0.12, 0.08, 0.04)
NVFP4_TENSOR_SCALE = 2.0 ** -9


def draw_w0_nvfp4(workload: str, seed: int, band: int, layer_type: str, family: str, N: int, K: int):
    """(codes uint8[N, K/2], scale bytes uint8[N, K/16], tensor scale) of an
    NVFP4 W0; element 2i of a row in the low nibble of byte i."""
    assert K % 16 == 0
    g = _gen(workload, seed, "W0nvfp4", band, layer_type, family)
    mag = torch.multinomial(torch.tensor(NVFP4_MAG_WEIGHTS), N * K, replacement=True, generator=g)
    sign = torch.randint(0, 2, (N * K,), generator=g)
    nib = (mag + 8 * sign).to(torch.uint8).reshape(N, K)
    codes = nib[:, 0::2] | (nib[:, 1::2] << 4)
    scales = torch.randint(0x30, 0x50, (N, K // 16), generator=g).to(torch.uint8)
    return codes.contiguous(), scales, NVFP4_TENSOR_SCALE


def draw_x(workload: str, seed: int, M: int, K: int, tag="x") -> torch.Tensor:
    return normal_bf16((M, K), 1.0, workload, seed, tag, M, K)


def bf16_bits(t: torch.Tensor):
    """Raw uint16 view (numpy) of a CPU bf16 tensor."""
    import numpy as np

    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------ workloads -----
@dataclass
class Proj:
    family: str
    W0: torch.Tensor
    s: torch.Tensor
    U: torch.Tensor
    V: torch.Tensor

    @property
    def N(self):
        return self.W0.shape[0]

    @property
    def K(self):
        return self.W0.shape[1]

    @property
    def r(self):
        return self.U.shape[1]


@dataclass
class Call:
    """One forward call: P projections (P > 1: stacked) sharing one x."""
    layer: int
    projs: list
    x: torch.Tensor = field(default=None)


def tiny_band(seed: int = 0):
    """Tiny single band: G=2 layers sharing one W0 of 256x128; rank 4; x 4x128.
    Returns a list of two Calls (one per layer), both on the same x."""
    wl = "tiny"
    N, K, r, M = 256, 128, 4, 4
    W0 = draw_w0(wl, seed, 0, "all", "w", N, K)
    x = draw_x(wl, seed, M, K)
    calls = []
    for layer in range(2):
        s, U, V = draw_delta(wl, seed, layer, "w", N, K, r)
        calls.append(Call(layer, [Proj("w", W0, s, U, V)], x))
    return calls


def gemma3_sweep(seed: int, G: int, r: int, M: int, layers=None, stacked=True,
                 workload="gemma3_1b"):
    """Gemma-3-1B-shaped projections: one Call per (layer, stack).  W0 is shared
    per (band, family) with contiguous bands.  x is drawn per (M, K)."""
    L = GEMMA3_1B_LAYERS
    layers = range(L) if layers is None else layers
    w0_cache = {}
    xs = {}
    calls = []
    stacks = GEMMA3_1B_STACKS if stacked else [(f,) for f in GEMMA3_1B_FAMILIES]
    for l in layers:
        b = contiguous_band(l, L, G)
        for stack in stacks:
            projs = []
            for fam in stack:
                N, K = GEMMA3_1B_FAMILIES[fam]
                key = (b, fam)
                if key not in w0_cache:
                    w0_cache[key] = draw_w0(workload, seed, b, "all", fam, N, K)
                s, U, V = draw_delta(workload, seed, l, fam, N, K, r)
                projs.append(Proj(fam, w0_cache[key], s, U, V))
            K = projs[0].K
            if K not in xs:
                xs[K] = draw_x(workload, seed, M, K)
            calls.append(Call(l, projs, xs[K]))
    return calls


def gemma4_calls(seed: int, r: int, M: int, layers, stacked=True, families=None,
                 workload="gemma4_31b"):
    """Gemma-4-31B-shaped projections for the given layers.  W0 is shared per
    (band, layer_type, family) for attention and per (band, family) for the MLP."""
    L, G = GEMMA4_31B_LAYERS, GEMMA4_31B_BANDS
    w0_cache = {}
    xs = {}
    calls = []
    for l in layers:
        lt = gemma4_layer_type(l)
        b = contiguous_band(l, L, G)
        fams = gemma4_families(lt)
        stacks = gemma4_stacks(lt) if stacked else [(f,) for f in fams]
        for stack in stacks:
            if families is not None and not any(f in families for f in stack):
                continue
            projs = []
            for fam in stack:
                N, K = fams[fam]
                group = "mlp" if fam in GEMMA4_31B_MLP else lt
                key = (b, group, fam)
                if key not in w0_cache:
                    w0_cache[key] = draw_w0(workload, seed, b, group, fam, N, K)
                s, U, V = draw_delta(workload, seed, l, fam, N, K, r)
                projs.append(Proj(fam, w0_cache[key], s, U, V))
            K = projs[0].K
            if (M, K) not in xs:
                xs[(M, K)] = draw_x(workload, seed, M, K)
            calls.append(Call(l, projs, xs[(M, K)]))
    return calls


def random_case(seed: int, M: int, N: int, K: int, r: int, P: int = 1):
    """A generic seeded case (ragged shapes for parity tests)."""
    wl = "case"
    projs = []
    for p in range(P):
        Np = N if isinstance(N, int) else N[p]
        rp = r if isinstance(r, int) else r[p]
        W0 = draw_w0(wl, seed, p, "all", f"f{p}", Np, K)
        s, U, V = draw_delta(wl, seed, p, f"f{p}", Np, K, rp)
        projs.append(Proj(f"f{p}", W0, s, U, V))
    x = draw_x(wl, seed, M, K)
    return Call(0, projs, x)


# ------------------------------------------------------- device draws -------
def device_bundle(N: int, K: int, r: int, *key, device="cuda"):
    """(W0, s, U, V) drawn directly on `device` with the distributions above
    (W0, U, V ~ N(0, 0.02) bf16, s ~ U(0.9, 1.1) fp32) from a generator seeded
    by the key: for timing runs, where drawing hundreds of MB on the CPU would
    dominate.  A different random stream from the CPU draws."""
    g = torch.Generator(device=device)
    g.manual_seed(subseed("device", *key))
    W0 = (torch.randn(N, K, generator=g, device=device) * W_STD).to(torch.bfloat16)
    s = torch.rand(N, generator=g, device=device) * (S_HI - S_LO) + S_LO
    U = (torch.randn(N, r, generator=g, device=device) * W_STD).to(torch.bfloat16) if r else None
    V = (torch.randn(K, r, generator=g, device=device) * W_STD).to(torch.bfloat16) if r else None
    return W0, s, U, V


def device_x(M: int, K: int, *key, device="cuda"):
    """x ~ N(0, 1) bf16 drawn on `device` (see device_bundle)."""
    g = torch.Generator(device=device)
    g.manual_seed(subseed("device-x", *key))
    return torch.randn(M, K, generator=g, device=device).to(torch.bfloat16)


def device_nvfp4_bundle(N: int, K: int, r: int, *key, device="cuda"):
    """(codes N x K/2 uint8, scale bytes N x K/16 uint8, tensor scale, s, U, V)
    of an NVFP4 projection drawn on `device` for timing runs: uniformly random
    code bytes, scale bytes in 0x30 .. 0x4F (E4M3 0.5 .. 15), the tensor scale
    of draw_w0_nvfp4; s, U, V as device_bundle."""
    g = torch.Generator(device=device)
    g.manual_seed(subseed("device-nvfp4", *key))
    codes = torch.randint(0, 256, (N, K // 2), generator=g, device=device, dtype=torch.uint8)
    scales = torch.randint(0x30, 0x50, (N, K // 16), generator=g, device=device, dtype=torch.uint8)
    s = torch.rand(N, generator=g, device=device) * (S_HI - S_LO) + S_LO
    U = (torch.randn(N, r, generator=g, device=device) * W_STD).to(torch.bfloat16) if r else None
    V = (torch.randn(K, r, generator=g, device=device) * W_STD).to(torch.bfloat16) if r else None
    return codes, scales, NVFP4_TENSOR_SCALE, s, U, V

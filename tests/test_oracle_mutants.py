"""The forward pins must catch a plausible mistake in the oracle.

Each mutant is a copy of the oracle's C source with one planted error: a
dropped or mis-scaled term, a sign flip, a transposed or mis-indexed operand,
a short loop.  Every mutant is built with gcc and must fail at least one of
the pins in test_oracle_forward (the unmodified source must pass them all).
Nothing here runs on a GPU; the mistakes are planted in the oracle only.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_forward as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "wl_oracle.c")

# (what is replaced in the factored forward, replacement)
MUTANTS = {
    "drop_delta": ("y[m * N + n] = (double)s[n] * z + d;", "y[m * N + n] = (double)s[n] * z;"),
    "scale_on_delta": ("y[m * N + n] = (double)s[n] * z + d;", "y[m * N + n] = (double)s[n] * (z + d);"),
    "delta_sign": ("y[m * N + n] = (double)s[n] * z + d;", "y[m * N + n] = (double)s[n] * z - d;"),
    "drop_scale": ("y[m * N + n] = (double)s[n] * z + d;", "y[m * N + n] = z + d;"),
    "v_transposed": ("acc += widen_bf16(V[k * r + j]) * widen_bf16(x[m * K + k]);",
                     "acc += widen_bf16(V[j * K + k]) * widen_bf16(x[m * K + k]);"),
    "u_transposed": ("d += widen_bf16(U[n * r + j]) * T[m * r + j];",
                     "d += widen_bf16(U[j * N + n]) * T[m * r + j];"),
    "t_row_index": ("d += widen_bf16(U[n * r + j]) * T[m * r + j];",
                    "d += widen_bf16(U[n * r + j]) * T[j];"),
    "w0_short_k": ("for (long k = 0; k < K; ++k)\n                z +=", "for (long k = 1; k < K; ++k)\n                z +="),
    "x_index_in_t": ("acc += widen_bf16(V[k * r + j]) * widen_bf16(x[m * K + k]);",
                     "acc += widen_bf16(V[k * r + j]) * widen_bf16(x[k]);"),
}


def _pin_calls():
    """Every forward pin with concrete arguments (parametrized ones expanded)."""
    calls = [pins.test_hand_computed_2x2_rank1, pins.test_hand_computed_rank2_asymmetric,
             pins.test_no_delta_unit_scale_is_plain_matmul, pins.test_scale_only_applies_to_shared_block,
             pins.test_linearity_and_rank_permutation, pins.test_decomposed_passthrough_reproduces_dense_matmul]
    for args in [(1, 5, 7, 3), (3, 4, 9, 1), (2, 6, 3, 4), (2, 3, 4, 0)]:
        calls.append(lambda a=args: pins.test_exact_small_integers_bruteforce(*a))
    for args in [(3, 37, 24, 5), (1, 8, 64, 16), (5, 19, 13, 7)]:
        calls.append(lambda a=args: pins.test_factored_equals_dense_effective_weight(*a))
    return calls


def _build(tmp_path, name, text):
    src = tmp_path / f"{name}.c"
    lib = tmp_path / f"{name}.so"
    src.write_text(text)
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                           "-o", str(lib), str(src)])
    L = ctypes.CDLL(str(lib))
    for fn in ("wl_oracle_forward", "wl_oracle_forward_dense"):
        getattr(L, fn).restype = ctypes.c_int
        getattr(L, fn).argtypes = [ctypes.c_void_p] * 6 + [ctypes.c_long] * 4
    return L


def _failures(monkeypatch, lib):
    """How many pins fail when the oracle's factored forward is `lib`'s."""
    monkeypatch.setattr(oracle, "forward",
                        lambda x, W0, s, U, V: oracle._run("wl_oracle_forward", x, W0, s, U, V, lib=lib))
    failed = 0
    for call in _pin_calls():
        try:
            call()
        except AssertionError:
            failed += 1
    monkeypatch.undo()
    return failed


def test_unmodified_source_passes_every_pin(tmp_path, monkeypatch):
    text = open(SRC).read()
    assert _failures(monkeypatch, _build(tmp_path, "original", text)) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(tmp_path, monkeypatch, name):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation site of {name} not found exactly once"
    lib = _build(tmp_path, name, text.replace(old, new))
    assert _failures(monkeypatch, lib) > 0, f"no pin catches the mutant {name}"


# ----------------------------------------------------- decomposition oracle --
import types  # noqa: E402

import test_oracle_decompose as dpins  # noqa: E402

DSRC = os.path.join(os.path.dirname(oracle.__file__), "decompose.py")

DMUTANTS = {
    "first_layer_not_mean": ("W0[b] = np.mean(W[members], axis=0)", "W0[b] = W[members[0]]"),
    "scale_inverted": ("num / np.where(den > 0, den, 1.0)", "np.where(den > 0, den, 1.0) / np.where(num != 0, num, 1.0)"),
    "residual_unscaled": ("R = W[l] - s[l][:, None] * w0", "R = W[l] - w0"),
    "sigma_dropped": ("U[l, :, :kk] = P[:, :kk] * sig[:kk]", "U[l, :, :kk] = P[:, :kk]"),
    "truncation_short": ("kk = min(r, sig.shape[0])", "kk = min(r, sig.shape[0]) - 1"),
    "v_from_left_factor": ("V[l, :, :kk] = Qt[:kk].T", "V[l, :, :kk] = Qt.T[:, -kk:] if kk else Qt[:0].T"),
    "bands_interleaved": ("return [(l * G) // L for l in range(L)]", "return [l % G for l in range(L)]"),
}


def _dpin_calls():
    calls = [dpins.test_band_mean_and_scalar_multiples, dpins.test_least_squares_residual_orthogonal_to_w0_rows,
             dpins.test_error_non_increasing_in_rank_and_eckart_young, dpins.test_factors_orthonormal_and_sigma_in_u,
             dpins.test_rank_beyond_matrix_is_zero_padded, dpins.test_explicit_interleaved_bands]
    for r in dpins.GOLDEN["passthrough_error"]["ranks"]:
        calls.append(lambda rr=r: dpins.test_passthrough_is_exact_for_every_rank(rr))
    return calls


def _dfailures(monkeypatch, text):
    mod = types.ModuleType("decompose_mutant")
    exec(compile(text, "decompose_mutant.py", "exec"), mod.__dict__)
    monkeypatch.setattr(oracle, "decompose", mod.decompose)
    monkeypatch.setattr(oracle, "relative_frobenius_error", mod.relative_frobenius_error)
    failed = 0
    for call in _dpin_calls():
        try:
            call()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    monkeypatch.undo()
    return failed


def test_decompose_unmodified_passes_every_pin(monkeypatch):
    assert _dfailures(monkeypatch, open(DSRC).read()) == 0


@pytest.mark.parametrize("name", sorted(DMUTANTS))
def test_decompose_planted_mistake_is_caught(monkeypatch, name):
    """Mistakes are planted in the mean decomposition (the code before the ALS
    refinement, which repeats some of its steps)."""
    old, new = DMUTANTS[name]
    text = open(DSRC).read()
    cut = text.index("\ndef theta_objective")
    head, tail = text[:cut], text[cut:]
    assert head.count(old) == 1, f"mutation site of {name} not found exactly once"
    assert _dfailures(monkeypatch, head.replace(old, new) + tail) > 0, f"no pin catches the mutant {name}"


# ----------------------------------------------------------------- NVFP4 ---
# The NVFP4 pins (test_oracle_nvfp4) must catch a plausible mistake in the
# encoding oracle: wrong nibble order, exponent bias or subnormal step, ties
# away from zero, a dropped sign, a mis-scaled block or tensor scale, or a
# forward that drops a term.
import test_oracle_nvfp4 as npins  # noqa: E402

NSRC = os.path.join(os.path.dirname(oracle.__file__), "nvfp4.py")

NMUTANTS = {
    "nibble_order": ("return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)",
                     "return (c[:, 1::2] | (c[:, 0::2] << 4)).astype(np.uint8)"),
    "e4m3_bias": ("np.exp2(e - 7.0)", "np.exp2(e - 8.0)"),
    "e4m3_subnormal_step": ("m / 8.0 * 2.0 ** -6", "m / 8.0 * 2.0 ** -7"),
    "e2m1_subnormal_step": ("(c & 1) * 0.5 if (c >> 1) == 0", "(c & 1) * 0.25 if (c >> 1) == 0"),
    "ties_away_from_zero": ("pick_hi = (dhi < dlo) | ((dhi == dlo) & even[hi])", "pick_hi = dhi <= dlo"),
    "sign_dropped": ("return (idx + np.where(np.signbit(v), 8, 0)).astype(np.uint8)",
                     "return idx.astype(np.uint8)"),
    "block_scale_over_4": ("sbytes = e4m3_encode(bmax / (E2M1_MAX * tensor_scale))",
                           "sbytes = e4m3_encode(bmax / (4.0 * tensor_scale))"),
    "tensor_scale_without_6": ("np.float32(amax / (E2M1_MAX * E4M3_MAX))", "np.float32(amax / E4M3_MAX)"),
    "dequant_drops_tensor_scale": ("return (vals * e4m3_decode(sbytes)[:, :, None] * tensor_scale).reshape(N, K)",
                                   "return (vals * e4m3_decode(sbytes)[:, :, None]).reshape(N, K)"),
    "forward_drops_scale": ("y = f64(s)[None, :] * (X @ W0.T)", "y = X @ W0.T"),
    "forward_drops_delta": ("y = y + (X @ Vf) @ Uf.T", "y = y"),
}


def _npin_calls():
    calls = [npins.test_e4m3_decode_matches_torch, npins.test_e4m3_encode_matches_torch_rounding,
             npins.test_e2m1_rounding_brute_force, npins.test_e2m1_table_shape, npins.test_golden_blocks,
             npins.test_lossless_round_trip, npins.test_bytes_per_element,
             npins.test_forward_matches_the_c_oracle_on_an_exact_weight]
    for std in (0.02, 1.0, 300.0):
        calls.append(lambda sd=std: npins.test_rounding_error_bound(sd))
    return calls


def _nfailures(monkeypatch, text):
    mod = types.ModuleType("nvfp4_mutant")
    exec(compile(text, "nvfp4_mutant.py", "exec"), mod.__dict__)
    monkeypatch.setattr(npins, "nvfp4", mod)
    failed = 0
    for call in _npin_calls():
        try:
            call()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    monkeypatch.undo()
    return failed


def test_nvfp4_unmodified_passes_every_pin(monkeypatch):
    assert _nfailures(monkeypatch, open(NSRC).read()) == 0


@pytest.mark.parametrize("name", sorted(NMUTANTS))
def test_nvfp4_planted_mistake_is_caught(monkeypatch, name):
    old, new = NMUTANTS[name]
    text = open(NSRC).read()
    assert text.count(old) == 1, f"mutation site of {name} not found exactly once"
    assert _nfailures(monkeypatch, text.replace(old, new)) > 0, f"no pin catches the mutant {name}"

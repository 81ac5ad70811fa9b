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

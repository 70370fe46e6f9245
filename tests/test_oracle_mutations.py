"""The oracle's pins must be strong enough to catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (a dropped
term, a wrong sign or index, a transposed operand, an off-by-one mask, the
wrong logarithm), compiles the copy into a temporary directory, swaps it in,
and runs the pin tests: at least one pin must fail.  The numpy parts (KV-cache
decode, RoPE + QK-norm prologue) get the same treatment from a mutated copy of
their Python source.  Nothing here touches the
committed oracle or the GPU.
"""
import ast
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

MUTATIONS = {
    "scores_without_scale": ("s[j] = scale * acc;", "s[j] = acc;"),
    "mask_drops_diagonal": ("if (j > i) return 0;", "if (j >= i) return 0;"),
    "doc_mask_off_by_one": ("j < doc_row[i]) return 0;", "j <= doc_row[i]) return 0;"),
    "window_off_by_one": ("j <= i - window) return 0;", "j < i - window) return 0;"),
    "window_ignored": ("if (window > 0 && j <= i - window) return 0;", ""),
    "lse_in_log2": ("return m + log(z);", "return m + log2(z);"),
    "jacobian_sign": ("(j == kk ? p[j] : 0.0) - p[j] * p[kk]", "(j == kk ? p[j] : 0.0) + p[j] * p[kk]"),
    "jacobian_drops_diag": ("(j == kk ? p[j] : 0.0) - p[j] * p[kk]", "- p[j] * p[kk]"),
    "dk_uses_key": ("dkj[c] += g * qi[c];", "dkj[c] += g * kj[c];"),
    "grad_without_scale": ("const double g = scale * ds[j];", "const double g = ds[j];"),
    "dv_transposed": ("dvj[c] += p[j] * doi[c];", "dvj[c] += p[j] * vj[c];"),
    "dp_uses_query": ("acc += doi[c] * vj[c];", "acc += doi[c] * qi[c];"),
    "output_unnormalised": ("for (int j = 0; j <= i; ++j) p[j] /= z;", ""),
}

PIN_TESTS = [
    (pins.test_single_token_closed_form, {}),
    (pins.test_first_row_sees_only_itself, {}),
    (pins.test_two_token_closed_form, {}),
    (pins.test_uniform_values_give_that_value, {}),
    (pins.test_probability_rows, {}),
    (pins.test_probability_rows_with_documents, {}),
    (pins.test_gradient_sums, {}),
    (pins.test_central_finite_differences, {"T": 3, "d": 4, "with_doc": False}),
    (pins.test_central_finite_differences, {"T": 5, "d": 2, "with_doc": True}),
    (pins.test_against_torch_sdpa_fp64, {"B": 1, "H": 2, "T": 64, "d": 32, "with_doc": False}),
    (pins.test_against_torch_sdpa_fp64, {"B": 2, "H": 1, "T": 60, "d": 16, "with_doc": True}),
    (pins.test_window_of_one_key_closed_form, {}),
    (pins.test_window_probability_rows, {"w": 3}),
    (pins.test_window_against_torch_sdpa_fp64, {"T": 64, "d": 32, "w": 16, "with_doc": False}),
]


def _compile_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mutant.so"
    subprocess.run(["gcc", "-O1", "-std=c99", "-fopenmp", "-fPIC", "-shared", "-o", str(so),
                    str(path), "-lm"], check=True)
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path, monkeypatch):
    old, new = MUTATIONS[name]
    so = _compile_mutant(tmp_path, old, new)
    real = oracle._load()
    lib = ctypes.CDLL(so)
    for fn in ("oracle_attn_fwd", "oracle_attn_bwd", "oracle_attn_fwd_window",
               "oracle_attn_bwd_window"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = ctypes.c_int
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    for fn, kw in PIN_TESTS:
        try:
            fn(**kw)
        except AssertionError:
            caught.append(fn.__name__)
    assert caught, f"no pin caught the planted mistake {name!r}"


# ---------------------------------------------------------- the numpy parts of the oracle
# The KV-cache decode and the RoPE + QK-norm prologue are written in numpy inside
# oracle/__init__.py.  Each case plants one mistake in a copy of that source, rebuilds the
# affected functions from the copy, swaps them into the oracle module and runs the pins.


PY_SRC = oracle.__file__
PY_FUNCS = ("_f64", "_rope_angles", "_rope", "qk_prologue_forward", "qk_prologue_backward",
            "decode_forward")

PY_MUTATIONS = {
    "decode_sees_one_key_too_few": ("n = L - Tq + t + 1 ", "n = L - Tq + t "),
    "decode_sees_whole_cache": ("n = L - Tq + t + 1 ", "n = L "),
    "decode_without_scale": ("s = scale * (kc[b, :n, h, :] @ q[b, t, h, :])",
                             "s = (kc[b, :n, h, :] @ q[b, t, h, :])"),
    "decode_lse_in_log2": ("lse[b, h, t] = m + np.log(z)", "lse[b, h, t] = m + np.log2(z)"),
    "decode_unnormalised": ("o[b, t, h] = (w / z) @ vc", "o[b, t, h] = w @ vc"),
    "decode_first_token_query": ("@ q[b, t, h, :])", "@ q[b, 0, h, :])"),
    "rope_adjacent_pairs": ("x1, x2 = x[..., :h], x[..., h:]", "x1, x2 = x[..., 0::2], x[..., 1::2]"),
    "rope_not_a_rotation": ("-x1 * s + x2 * cos", "x1 * s + x2 * cos"),
    "rope_frequency_exponent": ("theta = base ** (-2.0 * i / d)", "theta = base ** (-i / d)"),
    "rope_positions_from_one": ("ang = np.arange(T, dtype=np.float64)[:, None]",
                                "ang = np.arange(1, T + 1, dtype=np.float64)[:, None]"),
    "norm_without_eps": ("r = np.sqrt(np.mean(u * u, axis=-1, keepdims=True) + eps)\n    return",
                         "r = np.sqrt(np.mean(u * u, axis=-1, keepdims=True))\n    return"),
    "norm_sum_not_mean": ("r = np.sqrt(np.mean(u * u, axis=-1, keepdims=True) + eps)\n    return",
                          "r = np.sqrt(np.sum(u * u, axis=-1, keepdims=True) + eps)\n    return"),
    "forward_drops_gain": ("return gain * u / r", "return u / r"),
    "backward_drops_projection": ("du = (gain / r) * (dz - u * s / (d * r * r))",
                                  "du = (gain / r) * dz"),
    "backward_projection_without_d": ("du = (gain / r) * (dz - u * s / (d * r * r))",
                                      "du = (gain / r) * (dz - u * s / (r * r))"),
    "backward_rotates_forward": ("return _rope(du, cos, sin, inverse=True)",
                                 "return _rope(du, cos, sin)"),
    "backward_drops_gain": ("du = (gain / r) * (dz", "du = (1.0 / r) * (dz"),
}

PY_PIN_TESTS = [
    (pins.test_decode_is_the_last_rows_of_causal_attention, {"B": 1, "H": 2, "Tq": 1, "L": 1, "d": 4}),
    (pins.test_decode_is_the_last_rows_of_causal_attention, {"B": 1, "H": 2, "Tq": 5, "L": 20, "d": 4}),
    (pins.test_decode_single_cached_token, {}),
    (pins.test_decode_against_torch_sdpa_fp64, {}),
    (pins.test_prologue_against_torch_fp64, {}),
    (pins.test_prologue_position_zero_is_plain_rms_norm, {}),
    (pins.test_prologue_rotation_keeps_rms_and_commutes_with_the_norm, {}),
    (pins.test_prologue_scores_depend_on_relative_position_only, {}),
    (pins.test_prologue_finite_differences, {}),
]


def _mutant_functions(old, new):
    src = open(PY_SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    tree = ast.parse(src.replace(old, new))
    keep = [n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name in PY_FUNCS]
    assert {n.name for n in keep} == set(PY_FUNCS)
    ns = {"np": oracle.np}
    exec(compile(ast.Module(body=keep, type_ignores=[]), "mutant_oracle", "exec"), ns)
    return {name: ns[name] for name in PY_FUNCS}


def test_python_mutation_anchors_are_unique():
    src = open(PY_SRC).read()
    for name, (old, _) in PY_MUTATIONS.items():
        assert src.count(old) == 1, name


@pytest.mark.parametrize("name", sorted(PY_MUTATIONS))
def test_planted_mistake_in_numpy_oracle_is_caught(name, monkeypatch):
    old, new = PY_MUTATIONS[name]
    for fn_name, fn in _mutant_functions(old, new).items():
        monkeypatch.setattr(oracle, fn_name, fn)
    caught = []
    for fn, kw in PY_PIN_TESTS:
        try:
            with np.errstate(all="ignore"):
                fn(**kw)
        except (AssertionError, ValueError, IndexError):
            caught.append(fn.__name__)
    assert caught, f"no pin caught the planted mistake {name!r}"


def test_unmutated_numpy_oracle_passes_every_pin(monkeypatch):
    """The harness itself: the functions rebuilt from the unchanged source pass all pins."""
    for fn_name, fn in _mutant_functions("def ", "def ").items():
        monkeypatch.setattr(oracle, fn_name, fn)
    for fn, kw in PY_PIN_TESTS:
        fn(**kw)


# ------------------------------------------------- the FP8 (e4m3) forward oracle (numpy)

from tests import test_oracle_fp8 as fp8pins  # noqa: E402

FP8_FUNCS = ("e4m3_decode", "_e4m3_table", "e4m3_encode", "e4m3_round", "fp8_dequantize",
             "fp8_weight_error_bound", "fp8_attention_forward", "fp8_attention_simulated")

FP8_MUTATIONS = {
    "e4m3_exponent_bias_8": ("np.exp2(e.astype(np.float64) - 7)", "np.exp2(e.astype(np.float64) - 8)"),
    "e4m3_subnormal_scale": ("m / 8.0 * 2.0 ** -6", "m / 8.0 * 2.0 ** -7"),
    "e4m3_ties_away_from_zero": ("((d_hi == d_lo) & (codes[hi] % 2 == 0))", "(d_hi == d_lo)"),
    "dequantize_ignores_descale": ("return float(descale) * e4m3_decode", "return e4m3_decode"),
    "weights_not_scaled_before_rounding": ("qw = e4m3_round(p_scale * r) / p_scale", "qw = e4m3_round(r)"),
    "weights_normalised_before_rounding": ("r = p / p.max(axis=1, keepdims=True)\n            qw",
                                           "r = p\n            qw"),
    "simulated_exact_sum": ("o[b, h] = (qw @ v[b, h]) / qw.sum(axis=1, keepdims=True)",
                            "o[b, h] = (qw @ v[b, h]) / r.sum(axis=1, keepdims=True)"),
    "bound_half_an_ulp_too_small": ("(2.0 ** -4 + 2.0 ** -14) * r", "(2.0 ** -5 + 2.0 ** -14) * r"),
    "bound_deviation_from_zero": ("np.abs(vb[None, :, :] - o[b, h, i0:i1, None, :])",
                                  "np.abs(vb[None, :, :] + 0 * o[b, h, i0:i1, None, :])"),
}


def _fp8_mutant(old, new):
    src = open(PY_SRC).read()
    tree = ast.parse(src.replace(old, new))
    keep = [n for n in tree.body if isinstance(n, ast.FunctionDef) and n.name in FP8_FUNCS]
    assert {n.name for n in keep} == set(FP8_FUNCS)
    ns = dict(vars(oracle))
    ns["_E4M3_POS"] = None
    exec(compile(ast.Module(body=keep, type_ignores=[]), "mutant_oracle", "exec"), ns)
    return ns


def _fp8_pins():
    out = []
    for name in dir(fp8pins):
        fn = getattr(fp8pins, name)
        if name.startswith("test_") and callable(fn):
            params = fn.__code__.co_varnames[:fn.__code__.co_argcount]
            out.append((fn, {"seed": 10} if "seed" in params else {}))
    return out


def test_fp8_mutation_anchors_are_unique():
    src = open(PY_SRC).read()
    for name, (old, _) in FP8_MUTATIONS.items():
        assert src.count(old) == 1, name


@pytest.mark.parametrize("name", sorted(FP8_MUTATIONS))
def test_planted_mistake_in_fp8_oracle_is_caught(name, monkeypatch):
    old, new = FP8_MUTATIONS[name]
    ns = _fp8_mutant(old, new)
    for fn_name in FP8_FUNCS:
        monkeypatch.setattr(oracle, fn_name, ns[fn_name])
    monkeypatch.setattr(oracle, "_E4M3_POS", None)
    caught = []
    for fn, kw in _fp8_pins():
        try:
            with np.errstate(all="ignore"):
                fn(**kw)
        except (AssertionError, ValueError, IndexError):
            caught.append(fn.__name__)
    assert caught, f"no pin caught the planted mistake {name!r}"


def test_unmutated_fp8_oracle_passes_every_pin(monkeypatch):
    ns = _fp8_mutant("def ", "def ")
    for fn_name in FP8_FUNCS:
        monkeypatch.setattr(oracle, fn_name, ns[fn_name])
    monkeypatch.setattr(oracle, "_E4M3_POS", None)
    for fn, kw in _fp8_pins():
        fn(**kw)

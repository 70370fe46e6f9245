"""The oracle's pins must be strong enough to catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (a dropped
term, a wrong sign or index, a transposed operand, an off-by-one mask, the
wrong logarithm), compiles the copy into a temporary directory, swaps it in,
and runs the pin tests: at least one pin must fail.  Nothing here touches the
committed oracle or the GPU.
"""
import ctypes
import os
import subprocess

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

"""Planted mistakes: each test copies the oracle's C source, plants one
plausible mistake (a dropped term, a wrong sign, an off-by-one index, a
transposed operand, the wrong logarithm), builds the copy, and checks that the
pins in test_oracle_pins.py reject it.  Everything runs on the CPU."""
import os
import shutil
import subprocess

import pytest

import test_oracle_block_sparse as bsp
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "oracle", "attention_oracle.c")

# (name, original text, planted text)
MUTANTS = [
    ("jacobian-sign", "double ds = s[j] * dp[j] - s[j] * c;", "double ds = s[j] * dp[j] + s[j] * c;"),
    ("key-jacobian-dropped-p", "double ds = p * dp - p * c[i];", "double ds = p * dp - c[i];"),
    ("dq-scale-dropped", "dq_out[t] *= scale;", "dq_out[t] *= 1.0;"),
    ("dk-scale-dropped", "dk_out[t] *= scale;", "dk_out[t] *= 1.0;"),
    ("causal-off-by-one", "long n = i + 1;", "long n = i + 2;"),
    ("key-loop-off-by-one", "long i0 = causal ? j : 0;", "long i0 = causal ? j + 1 : 0;"),
    ("log2-instead-of-ln", "return m + log(z);", "return m + log2(z);"),
    ("dv-transposed-operand", "dv_out[t] += p * doi[t];", "dv_out[t] += p * qi[t];"),
    ("dp-wrong-operand", "dp[j] = dot(doi, vh + j * d, d);", "dp[j] = dot(qi, vh + j * d, d);"),
    ("reversed-dot", "s += a[t] * b[t];", "s += a[t] * b[d - 1 - t];"),
    ("forward-unnormalised", "double p = exp(s[j] - L);\n                    const double* vj",
     "double p = exp(s[j]);\n                    const double* vj"),
    ("scale-dropped-in-scores", "s[j] = scale * dot(qi, kh + j * d, d);",
     "s[j] = dot(qi, kh + j * d, d);"),
]


def _pin_suite(o):
    yield lambda: pins.test_worked_example_causal_n2_d2(o)
    yield lambda: pins.test_causal_row0_closed_form(o, 8)
    yield lambda: pins.test_identical_keys_prefix_mean(o, True)
    yield lambda: pins.test_identity_values_expose_probabilities(o, True)
    yield lambda: pins.test_shift_invariances(o, True)
    yield lambda: pins.test_gradient_invariants(o, True)
    yield lambda: pins.test_finite_differences(o, 3, 4, True)
    yield lambda: pins.test_against_torch_sdpa_float64(o, 1, 2, 17, 8, True)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_planted_mistake(oracle_mod, tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    cfile = tmp_path / "mutant.c"
    cfile.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(cfile),
                    "-o", str(so), "-lm"], check=True)
    caught = []
    oracle_mod._swap_library(str(so))
    try:
        for pin in _pin_suite(oracle_mod):
            try:
                pin()
            except (AssertionError, RuntimeError, FloatingPointError):
                caught.append(True)
    finally:
        oracle_mod._swap_library(None)
    assert caught, f"no pin caught the planted mistake {name}"


# Planted mistakes in the block-sparse functions, checked by the block-sparse pins.
BS_MUTANTS = [
    ("bs-causal-flip", "if (causal && j > i) return 0;", "if (causal && j >= i) return 0;"),
    ("bs-block-sizes-swapped", "return mask[(i / bq) * nbk + (j / bk)] != 0;",
     "return mask[(i / bk) * nbk + (j / bq)] != 0;"),
    ("bs-empty-row-lse", "lse[h * nq + i] = -INFINITY;", "lse[h * nq + i] = 0.0;"),
    ("bs-jacobian-dropped", "double ds = s[r] * dp[r] - s[r] * ci;", "double ds = s[r] * dp[r];"),
    ("bs-key-visibility-dropped",
     "if (!visible_bs(i, j, causal, mask, nbk, bq, bk)) continue;\n                    const double* qi",
     "const double* qi"),
    ("bs-dv-transposed-operand", "dvj[t] += p * doi[t];", "dvj[t] += p * qi[t];"),
]


def _bs_pin_suite(o):
    yield lambda: bsp.test_worked_example_block_sparse_n4_d2(o)
    yield lambda: bsp.test_all_ones_mask_is_dense(o, True)
    yield lambda: bsp.test_block_diagonal_is_blockwise_dense(o)
    yield lambda: bsp.test_against_torch_sdpa_with_element_mask(o, True, 3, 8, 4)
    yield lambda: bsp.test_against_torch_sdpa_with_element_mask(o, False, 0, 8, 8)
    yield lambda: bsp.test_rows_without_keys(o, True)
    yield lambda: bsp.test_finite_differences(o, True)


@pytest.mark.parametrize("name,old,new", BS_MUTANTS, ids=[m[0] for m in BS_MUTANTS])
def test_block_sparse_pins_reject_planted_mistake(oracle_mod, tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found once"
    cfile = tmp_path / "mutant.c"
    cfile.write_text(src.replace(old, new, 1))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", str(cfile),
                    "-o", str(so), "-lm"], check=True)
    caught = []
    oracle_mod._swap_library(str(so))
    try:
        for pin in _bs_pin_suite(oracle_mod):
            try:
                pin()
            except (AssertionError, RuntimeError, FloatingPointError):
                caught.append(True)
    finally:
        oracle_mod._swap_library(None)
    assert caught, f"no pin caught the planted mistake {name}"

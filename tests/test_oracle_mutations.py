"""The pins are sensitive: each plausible slip, planted in a private copy of
the oracle's C source and compiled on the CPU, makes at least one pin of
tests/test_oracle.py fail.  The real oracle is never modified."""
import importlib.util
import os
import shutil

import pytest

import test_oracle as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")

# (name, original text, planted text, pins expected to notice)
MUTATIONS = [
    ("flipped kernel rows",
     "long ih = p * g->sh - g->ph + r * g->dh;",
     "long ih = p * g->sh - g->ph + (g->R - 1 - r) * g->dh;",
     ["shifted_delta", "library", "numpy"]),
    ("wrong group of an output channel",
     "long gi = k / kpg;",
     "long gi = k % g->groups;",
     ["grouped", "library", "numpy"]),
    ("padding read as edge clamp",
     "if (ih < 0 || ih >= g->H) continue;",
     "if (ih < 0) ih = 0; if (ih >= g->H) ih = g->H - 1;",
     ["all_ones", "shifted_delta", "library"]),
    ("W index reads the H padding",
     "long iw = q * g->sw - g->pw + s * g->dw;",
     "long iw = q * g->sw - g->ph + s * g->dw;",
     ["axis_all_ones", "axis_shift", "axis_library"]),
    ("row index takes the W stride",
     "long ih = p * g->sh - g->ph + r * g->dh;",
     "long ih = p * g->sw - g->ph + r * g->dh;",
     ["axis_all_ones", "axis_shift", "axis_library"]),
    ("output size rounded up",
     "return span / stride + 1;",
     "return (span + stride - 1) / stride + 1;",
     ["sizes_closed_form", "sizes_pages"]),
    ("Bessel-corrected variance",
     "double var = ss / (double)M;",
     "double var = ss / (double)(M - 1);",
     ["gn_closed", "chain_library"]),
    ("eps outside the square root",
     "double inv = 1.0 / sqrt(var + eps);",
     "double inv = 1.0 / (sqrt(var) + eps);",
     ["gn_closed", "chain_library"]),
    ("scale applied before the biases",
     "a[o] = sigmoid_f64(z * sc);",
     "a[o] = sigmoid_f64((z - bc - be) * sc + bc + be);",
     ["bias_before_scale", "chain_library"]),
]

PINS = {
    "shifted_delta": lambda m: pins.test_shifted_delta_is_shift_with_zero_fill(m),
    "library": lambda m: pins.test_library_float64_conv(m),
    "numpy": lambda m: pins.test_numpy_restatement_tiny(m),
    "grouped": lambda m: pins.test_grouped_equals_concatenated_dense(m),
    "all_ones": lambda m: pins.test_all_ones_counts_in_bounds_taps(m),
    "sizes_closed_form": lambda m: pins.test_output_size_closed_form(m),
    "sizes_pages": lambda m: pins.test_output_sizes_from_pages(m),
    "gn_closed": lambda m: pins.test_chain_groupnorm_closed_forms(m),
    "chain_library": lambda m: pins.test_chain_matches_float64_library(m, 1.0, "random"),
    "bias_before_scale": lambda m: pins.test_chain_bias_before_scale(m),
    "axis_all_ones": lambda m: pins.test_per_axis_all_ones_counts_in_bounds_taps(m),
    "axis_shift": lambda m: pins.test_per_axis_shifted_delta_is_shift(m),
    "axis_library": lambda m: pins.test_per_axis_library_float64_conv(m),
}


def _mutated_oracle(tmp_path, original, planted):
    src = open(os.path.join(ORACLE_DIR, "oracle.c")).read()
    assert src.count(original) == 1, original
    d = tmp_path / "oracle_mut"
    d.mkdir()
    shutil.copy(os.path.join(ORACLE_DIR, "__init__.py"), d / "__init__.py")
    (d / "oracle.c").write_text(src.replace(original, planted))
    spec = importlib.util.spec_from_file_location(f"oracle_mut_{abs(hash(planted))}", d / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


@pytest.mark.parametrize("name,original,planted,expect", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_slip_is_caught(tmp_path, name, original, planted, expect):
    mod = _mutated_oracle(tmp_path, original, planted)
    caught = []
    for pin in expect:
        try:
            PINS[pin](mod)
        except (AssertionError, ValueError):
            caught.append(pin)
    assert caught, f"no pin noticed the planted slip '{name}'"


# slips planted in the float64 affine + clamp step of the Python wrapper
PY_MUTATIONS = [
    ("shift added before the scale",
     "y = y * s[None, :, None, None] + t[None, :, None, None]",
     "y = (y + t[None, :, None, None]) * s[None, :, None, None]",
     ["affine_bn"]),
    ("clamp bounds swapped",
     "y = np.minimum(np.maximum(y, float(lo)), float(hi))",
     "y = np.maximum(np.minimum(y, float(lo)), float(hi))",
     ["affine_relu6", "affine_bounds"]),
    ("scale ignored",
     "s = np.ones(K) if scale is None else _f32(scale).reshape(-1).astype(np.float64)",
     "s = np.ones(K)",
     ["affine_bn", "affine_relu6"]),
]

PINS.update({
    "affine_bn": lambda m: pins.test_affine_is_folded_batchnorm(m),
    "affine_relu6": lambda m: pins.test_affine_clamp_relu6_closed_form(m),
    "affine_bounds": lambda m: pins.test_affine_clamp_bounds_and_passthrough(m),
})


def _mutated_oracle_py(tmp_path, original, planted):
    src = open(os.path.join(ORACLE_DIR, "__init__.py")).read()
    assert src.count(original) == 1, original
    d = tmp_path / "oracle_mut_py"
    d.mkdir()
    shutil.copy(os.path.join(ORACLE_DIR, "oracle.c"), d / "oracle.c")
    (d / "__init__.py").write_text(src.replace(original, planted))
    spec = importlib.util.spec_from_file_location(f"oracle_mut_py_{abs(hash(planted))}", d / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


@pytest.mark.parametrize("name,original,planted,expect", PY_MUTATIONS, ids=[m[0] for m in PY_MUTATIONS])
def test_planted_affine_slip_is_caught(tmp_path, name, original, planted, expect):
    mod = _mutated_oracle_py(tmp_path, original, planted)
    caught = []
    for pin in expect:
        try:
            PINS[pin](mod)
        except (AssertionError, ValueError):
            caught.append(pin)
    assert caught, f"no pin noticed the planted slip '{name}'"

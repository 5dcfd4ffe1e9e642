"""The oracle's pins must catch a plausible slip anywhere in oracle.c.

Each case below plants one mistake in a copy of oracle.c (a wrong bit, bias,
index, stride, sign, a dropped term, a transposed operand), compiles the copy
with gcc into a temporary directory, and runs the pins of
test_oracle_pins.py against it.  At least one pin must fail for every
mutant.  Nothing here touches a GPU.
"""
import os

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

MUTATIONS = [
    ("e2m1 sign bit", "unsigned s = (code >> 3) & 1u;", "unsigned s = (code >> 2) & 1u;"),
    ("e2m1 subnormal", "mag = 0.5 * (double)m;", "mag = 1.0 * (double)m;"),
    ("e2m1 bias", "ldexp(1.0 + 0.5 * (double)m, (int)e - 1)", "ldexp(1.0 + 0.5 * (double)m, (int)e - 2)"),
    ("e4m3 bias", "ldexp(1.0 + (double)m / 8.0, (int)e - 7)", "ldexp(1.0 + (double)m / 8.0, (int)e - 8)"),
    ("e4m3 subnormal", "ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)"),
    ("e4m3 NaN set", "if (e == 15 && m == 7)", "if (e == 15)"),
    ("f16 subnormal", "ldexp((double)f, -24)", "ldexp((double)f, -25)"),
    ("f16 bias", "ldexp(1.0 + (double)f / 1024.0, (int)e - 15)", "ldexp(1.0 + (double)f / 1024.0, (int)e - 14)"),
    ("nibble order", "(k % 2 == 0) ? (byte & 0x0Fu) : (byte >> 4)", "(k % 2 == 0) ? (byte >> 4) : (byte & 0x0Fu)"),
    ("scale block size", "j->scales[n * (j->K / 16) + k / 16]", "j->scales[n * (j->K / 16) + k / 32]"),
    ("code row stride", "j->codes[n * (j->K / 2) + k / 2]", "j->codes[n * (j->K / 4) + k / 2]"),
    ("global scale divides", "* s * j->global_scale;", "* s / j->global_scale;"),
    ("fp8 channel index", "(double)j->channel_scale[n]", "(double)j->channel_scale[0]"),
    ("fp8 transposed operand", "j->codes[n * j->K + k]", "j->codes[k * j->N + n]"),
    ("dropped first term", "for (int64_t k = 0; k < j->K; ++k) {\n                double p",
     "for (int64_t k = 1; k < j->K; ++k) {\n                double p"),
    ("transposed output", "j->y[m * j->N + n] = acc;", "j->y[n * j->M + m] = acc;"),
    ("x row stride", "const double* xr = j->xd + m * j->K;", "const double* xr = j->xd + m;"),
    ("bound without abs", "mag += fabs(p);", "mag += p;"),
]


def _battery(orc):
    """Run the pins against one oracle build; return the names that failed."""
    checks = {
        "e2m1 table": lambda: pins.test_e2m1_matches_printed_table(orc),
        "e4m3 all": lambda: pins.test_e4m3_all_codes_match_torch_and_ml_dtypes(orc),
        "e4m3 special": lambda: pins.test_e4m3_matches_printed_special_values(orc),
        "f16 all": lambda: pins.test_f16_all_bit_patterns_match_numpy(orc),
        "nvfp4 exact a": lambda: pins.test_nvfp4_gemm_matches_exact_rationals(orc, 3, 4, 32, 3.0),
        "nvfp4 exact b": lambda: pins.test_nvfp4_gemm_matches_exact_rationals(orc, 8, 2, 48, 1.0 / 448.0),
        "fp8 exact": lambda: pins.test_fp8_gemm_matches_exact_rationals(orc, 4, 3, 40),
        "subnormal x": lambda: pins.test_nvfp4_subnormal_x_is_honoured(orc),
        "one hot": lambda: pins.test_one_hot_extracts_each_weight(orc),
        "numpy matmul": lambda: pins.test_second_implementation_numpy_matmul(orc),
        "fp8 numpy": lambda: pins.test_fp8_second_implementation(orc),
        "row independence": lambda: pins.test_row_independence_is_bitwise(orc),
    }
    failed = []
    for name, fn in checks.items():
        try:
            fn()
        except (AssertionError, ValueError, RuntimeError):
            failed.append(name)
    return failed


def test_unmutated_copy_passes_every_pin(tmp_path):
    out = oracle.compile_library(oracle.SOURCE, str(tmp_path / "liboracle_clean.so"), force=True)
    assert _battery(oracle.Oracle(out)) == []


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_planted_mistake_is_caught(tmp_path, name, old, new):
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert src.count(old) == 1, "mutation anchor must occur exactly once: %r" % old
    path = tmp_path / "oracle_mutant.c"
    path.write_text(src.replace(old, new))
    out = oracle.compile_library(str(path), str(tmp_path / "liboracle_mutant.so"), force=True)
    failed = _battery(oracle.Oracle(out))
    assert failed, "no pin caught the planted mistake: " + name


# ---------------------------------------------------------------------------
# silu_mul (numpy): each plausible slip must fail one of its pins
# ---------------------------------------------------------------------------

def _silu_mutants():
    def half(y):
        y = np.asarray(y, dtype=np.float64)
        F = y.shape[1] // 2
        return y[:, :F], y[:, F:]

    def exp_sign(y):            # e^+z instead of e^-z
        g, u = half(y)
        with np.errstate(over="ignore"):
            return g / (1.0 + np.exp(g)) * u

    def sigmoid_only(y):        # sigmoid(g) * u, the gate not multiplied back in
        g, u = half(y)
        with np.errstate(over="ignore"):
            return 1.0 / (1.0 + np.exp(-g)) * u

    def swapped(y):             # up and gate halves exchanged
        g, u = half(y)
        with np.errstate(over="ignore"):
            return u / (1.0 + np.exp(-u)) * g

    def no_mul(y):              # the up factor dropped
        g, _ = half(y)
        with np.errstate(over="ignore"):
            return g / (1.0 + np.exp(-g))

    def tanh_gelu(y):           # another activation in its place
        g, u = half(y)
        return 0.5 * g * (1.0 + np.tanh(0.7978845608 * (g + 0.044715 * g ** 3))) * u

    return [("exp sign", exp_sign), ("sigmoid only", sigmoid_only), ("swapped halves", swapped),
            ("no mul", no_mul), ("gelu", tanh_gelu)]


@pytest.mark.parametrize("name,fn", _silu_mutants(), ids=[n for n, _ in _silu_mutants()])
def test_silu_mul_pins_catch_mutant(name, fn, monkeypatch):
    monkeypatch.setattr(oracle, "silu_mul", fn)
    failed = 0
    for pin in (pins.test_silu_mul_closed_forms, pins.test_silu_mul_identities, pins.test_silu_mul_matches_torch_silu):
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1, name

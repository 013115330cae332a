"""Planted mistakes in the oracle must fail at least one pin (CPU only).

Each case copies one of the oracle's C files (aqlm_oracle.c, or
aqlm_encode_oracle.c for the encoding), changes one expression into a
plausible bug (a dropped term, a wrong sign, a swapped index, a transposed
operand, an off-by-one, a wrong rounding or tie rule), compiles the copy with
the other file into a temporary directory and runs the pins of
tests/oracle_pins.py against it.  Every planted change keeps all memory
accesses in bounds.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from oracle_pins import ALL_PINS

ORACLE_DIR = os.path.dirname(oracle.__file__)
INFER, ENCODE = "aqlm_oracle.c", "aqlm_encode_oracle.c"

MUTANTS = {
    "dequant_drops_scale": ("W[i * d_in + j * g + t] = s * sum;", "W[i * d_in + j * g + t] = sum;"),
    "codebooks_swapped": ("int64_t pos = (i * groups + j) * M + m;",
                          "int64_t pos = (i * groups + j) * M + (M - 1 - m);"),
    "codebook_transposed": ("sum += half_bits_to_double(codebooks[((int64_t)m * K + k) * g + t]);",
                            "sum += half_bits_to_double(codebooks[((int64_t)k * M + m) * g + t]);"),
    "gemv_wrong_sign": ("acc += (s * w[t]) *", "acc -= (s * w[t]) *"),
    "gemv_reversed_lanes": ("act_value(x, tau * d_in + j * g + t, is_bf16)",
                            "act_value(x, tau * d_in + j * g + (g - 1 - t), is_bf16)"),
    "gemv_drops_last_group": ("for (int64_t j = 0; j < groups; ++j) {\n                double w[64];",
                              "for (int64_t j = 0; j + 1 < groups; ++j) {\n                double w[64];"),
    "gemv_drops_second_codebook": ("for (int t = 0; t < g; ++t) w[t] += half_bits_to_double(cw[t]);",
                                   "for (int t = 0; t < g; ++t) w[t] = half_bits_to_double(cw[t]);"),
    "bf16_ties_away": ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) {",
                       "if (lower >= 0x8000u) {"),
    "bf16_fused_order": ("volatile float w = f * s;", "volatile float w = f * s + 0.0f * f + (float)1e-30;"),
    "half_subnormal_exponent": ("v = ldexp((double)frac, -24);", "v = ldexp((double)frac, -25);"),
    "bpp_scale_term": ("double scale_bits = (double)d_out * 16.0;", "double scale_bits = (double)d_out * 32.0;"),
    "bpp_codebook_term": ("double codebook_bits = (double)M * ldexp(1.0, B) * g * 16.0;",
                          "double codebook_bits = ldexp(1.0, B) * g * 16.0;"),
    # encoding
    "half_ties_away": (ENCODE, "double q = rint(ldexp(a, 11 - e));", "double q = round(ldexp(a, 11 - e));"),
    "scale_mean_abs": (ENCODE, "acc += (double)row[k] * (double)row[k];", "acc += fabs((double)row[k]);"),
    "nearest_ties_high": (ENCODE, "if (dk < bd) {", "if (dk <= bd) {"),
    "distance_drops_lane": (ENCODE, "for (int t = 0; t < 8; ++t) {\n        const double e",
                            "for (int t = 0; t < 7; ++t) {\n        const double e"),
    "distance_wrong_sign": (ENCODE, "(double)v[t] - (double)c[t]", "(double)v[t] + (double)c[t]"),
    "distance_not_squared": (ENCODE, "d += e * e;", "d += fabs(e);"),
    "runner_up_lost": (ENCODE, "            sd = bd;\n            bd = dk;", "            bd = dk;"),
    "update_off_by_one": (ENCODE, "(float)(sums[k * 8 + t] / (double)counts[k])",
                          "(float)(sums[k * 8 + t] / (double)(counts[k] + 1))"),
    "residual_not_subtracted": (ENCODE, "R[n * 8 + t] = R[n * 8 + t] - C[(int64_t)idx[n] * 8 + t];",
                                "R[n * 8 + t] = R[n * 8 + t] + 0.0f * C[(int64_t)idx[n] * 8 + t];"),
    "greedy_residual_kept": (ENCODE, "for (int t = 0; t < 8; ++t) r[t] = r[t] - Cm[best * 8 + t];",
                             "for (int t = 0; t < 8; ++t) r[t] = r[t] - 0.0f * Cm[best * 8 + t];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    case = MUTANTS[name]
    fname, old, new = case if len(case) == 3 else (INFER, *case)
    srcs = []
    for f in (INFER, ENCODE):
        text = open(os.path.join(ORACLE_DIR, f)).read()
        if f == fname:
            assert text.count(old) == 1, f"mutation site for {name} not found exactly once"
            text = text.replace(old, new)
        path = tmp_path / f
        path.write_text(text)
        srcs.append(str(path))
    lib_path = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", str(lib_path), *srcs, "-lm"], check=True)
    mutant = oracle._configure(ctypes.CDLL(str(lib_path)))
    saved = oracle._load()
    oracle._lib = mutant
    caught = None
    try:
        for pin in ALL_PINS:
            try:
                pin()
            except AssertionError:
                caught = pin.__name__
                break
    finally:
        oracle._lib = saved
    assert caught is not None, f"no pin caught the planted mistake {name}"

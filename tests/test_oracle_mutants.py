"""Planted mistakes in the oracle must fail at least one pin (CPU only).

Each case copies oracle/aqlm_oracle.c, changes one expression into a
plausible bug (a dropped term, a wrong sign, a swapped index, a transposed
operand, an off-by-one, a wrong rounding rule), compiles the copy into a
temporary directory and runs the pins of tests/oracle_pins.py against it.
Every planted change keeps all memory accesses in bounds.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
from oracle_pins import ALL_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "aqlm_oracle.c")

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
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib_path = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-o", str(lib_path), str(mutated), "-lm"], check=True)
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

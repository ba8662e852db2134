"""Plant a mistake in the oracle, on the CPU, and check that a pin catches it.

Each case edits one line of a copy of oracle/mxfp8_oracle.c (an off-by-one
scale exponent, ties to odd, a transposed weight index, a dropped bias, a
wrong scale index, overflow to NaN instead of saturation, a lost sign; for the
per-channel FP8 functions a wrong qmax, an amax over part of the row, a zero
row divided by its zero scale, a dropped weight scale; for NVFP4 a wrong
E2M1 exponent bias, ties to odd, g / 4 instead of g / 6, swapped nibbles,
a dropped global scale), builds the copy and
runs the pins against it; the pins must fail.  The real oracle is untouched.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "mxfp8_oracle.c")

MUTATIONS = {
    "scale_exponent_off_by_one": ("e = (ex - 1) - 8;", "e = ex - 8;"),
    "ties_to_odd": ("pick = (lo & 1) ? lo + 1 : lo;", "pick = (lo & 1) ? lo : lo + 1;"),
    "weight_transposed": ("wq[n * K + k]", "wq[k * N + n]"),
    "bias_dropped": ("acc += orc_f16_decode(bias[n]);", "acc += 0.0;"),
    "scale_index_wrong": ("xs[r * nb + k / 32]", "xs[r * nb + k % nb]"),
    "overflow_to_nan": ("if (a >= e4m3_mag[0x7E])\n        return sign | 0x7E;",
                        "if (a >= e4m3_mag[0x7E])\n        return sign | 0x7F;"),
    "sign_lost": ("return sign | (uint8_t)pick;", "return (uint8_t)pick;"),
    "subnormal_scale_wrong": ("mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);"),
    # per-channel FP8
    "rowwise_qmax_wrong": ("volatile float s = amax / 448.0f;", "volatile float s = amax / 447.0f;"),
    "rowwise_amax_half_row": ("for (int64_t k = 0; k < K; ++k) {\n        float a = fabsf(x[k]);",
                              "for (int64_t k = 0; k < K / 2; ++k) {\n        float a = fabsf(x[k]);"),
    "rowwise_zero_row_divides": ("if (s == 0.0f) {", "if (0) {"),
    "rowwise_weight_scale_dropped": ("acc = acc * (double)sx[r] * (double)sw[n];", "acc = acc * (double)sx[r];"),
    # NVFP4
    "e2m1_exponent_bias": ("ldexp(1.0 + 0.5 * m, E - 1)", "ldexp(1.0 + 0.5 * m, E - 2)"),
    "e2m1_ties_to_odd": ("(dc == db && (c & 1) == 0)", "(dc == db && (c & 1) == 1)"),
    "nvfp4_scale_over_4": ("volatile float gs = g / 6.0f;", "volatile float gs = g / 4.0f;"),
    "nvfp4_nibbles_swapped": ("codes[(16 * b + j) / 2] = (uint8_t)(lo | (hi << 4));",
                              "codes[(16 * b + j) / 2] = (uint8_t)(hi | (lo << 4));"),
    "nvfp4_global_scale_ignored": ("out[r * K + k] = orc_e2m1_decode(c) * orc_e4m3_decode(scales[r * (K / 16) + k / 16]) / (double)g;",
                                   "out[r * K + k] = orc_e2m1_decode(c) * orc_e4m3_decode(scales[r * (K / 16) + k / 16]);"),
}
PIN_FILES = ["test_oracle_pins.py", "test_oracle_pins_rowwise.py", "test_oracle_pins_nvfp4.py"]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mutated = src.replace(old, new)
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "m.c")
        so = os.path.join(td, "libm.so")
        open(c, "w").write(mutated)
        subprocess.run(["gcc", "-O1", "-std=c11", "-D_DEFAULT_SOURCE", "-fPIC", "-shared",
                        "-fopenmp", "-ffp-contract=off", "-o", so, c, "-lm"], check=True)
        env = dict(os.environ, ORACLE_LIB=so, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"]
                           + [os.path.join(ROOT, "tests", f) for f in PIN_FILES],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
        assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"

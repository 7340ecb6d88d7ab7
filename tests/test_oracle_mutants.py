"""Mutation check of the oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of oracle/bcq_oracle.c (a
flipped bit order, a dropped offset, a transposed scale index, ...), builds
it with gcc in a temporary directory, and runs tests/test_oracle_pins.py
against that build in a child process.  The pins must fail for every mutant;
the unmodified source must pass.  The committed oracle is never modified.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "bcq_oracle.c")
PINS = os.path.join(ROOT, "tests", "test_oracle_pins.py")

MUTANTS = {
    "bit_order_msb_first": ("(row_words[k / 32] >> (k % 32)) & 1u",
                            "(row_words[k / 32] >> (31 - k % 32)) & 1u"),
    "gemm_sign_swapped": ("v += a * (bit_at(row, k) ? 1.0 : -1.0);",
                          "v += a * (bit_at(row, k) ? -1.0 : 1.0);"),
    "offset_dropped": ("double v = z ? bcq_oracle_half_to_double(z[(size_t)n * G + g]) : 0.0;",
                       "double v = 0.0;"),
    "alpha_plane_major": ("aq[((size_t)n * G + g) * q + (i - 1)]",
                          "aq[((size_t)(i - 1) * N + n) * G + g]"),
    "alpha_wrong_precision": ("const uint16_t* aq = alpha[q - 1];",
                              "const uint16_t* aq = alpha[3];"),
    "plane_always_first": ("planes + ((size_t)(i - 1) * N + n) * KW",
                           "planes + ((size_t)0 * N + n) * KW"),
    "group_index_wrong": ("const int g = k / group;",
                          "const int g = (k / 8) % G;"),
    "lut_bit_reversed": ("(((b >> j) & 1) ? 1.0 : -1.0)",
                         "(((b >> (7 - j)) & 1) ? 1.0 : -1.0)"),
    "signed_sum_zero_one": ("const double s = bit_at(bits, k) ? 1.0 : -1.0;",
                            "const double s = bit_at(bits, k) ? 1.0 : 0.0;"),
    "half_bias_off": ("expo - 25", "expo - 24"),
    "group_sum_short": ("k < (g + 1) * group; ++k)",
                        "k < (g + 1) * group - 1; ++k)"),
    "x_row_ignored": ("const double* xm = xd + (size_t)m * K;",
                      "const double* xm = xd;"),
    "per_row_p_ignored": ("const double* wq = w + (size_t)(q - 1) * K;\n          const double* xm",
                          "const double* wq = w + (size_t)(used[4] ? 3 : q - 1) * K;\n          const double* xm"),
}


def _build(src_text, out_dir):
    c = os.path.join(out_dir, "m.c")
    so = os.path.join(out_dir, "libm.so")
    with open(c, "w", encoding="utf-8") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                    "-o", so, c, "-lm"], check=True)
    return so


def _run_pins(lib):
    env = dict(os.environ, BCQ_ORACLE_LIB=lib, OMP_NUM_THREADS="2")
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x",
                        "-p", "no:cacheprovider", PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    return r.returncode


@pytest.fixture(scope="module")
def source():
    with open(SRC, encoding="utf-8") as f:
        return f.read()


def test_unmodified_copy_passes(source):
    with tempfile.TemporaryDirectory() as d:
        assert _run_pins(_build(source, d)) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(source, name):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not unique"
    with tempfile.TemporaryDirectory() as d:
        assert _run_pins(_build(source.replace(old, new), d)) != 0

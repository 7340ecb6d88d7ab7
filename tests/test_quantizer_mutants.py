"""Mutation check of the quantiser oracle's pins (CPU only).

Each case plants one plausible mistake in a copy of oracle/quantizer.py (a
scale refit that skips the old planes, a flipped residual sign, the farthest
code instead of the nearest, a greedy scale over n - 1, ...) and runs
tests/test_quantizer_oracle.py against that copy in a child process
(BCQ_QUANTIZER_ORACLE).  The pins must fail for every mutant; the
unmodified copy must pass.  The committed oracle is never modified.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "quantizer.py")
PINS = os.path.join(ROOT, "tests", "test_quantizer_oracle.py")

MUTANTS = {
    # expansion refits only the new plane's scale, the old ones stay
    "expansion_new_scale_only": (
        "            alpha, _ = lsq(W, B, z)\n",
        "            a_new, _ = lsq(W - code_values(alpha, z, B[:, :-1]) + z[:, None], B[:, -1:], z)\n"
        "            alpha = np.concatenate([alpha, a_new], axis=1)\n"),
    "expansion_residual_sign_flipped": (
        "sign_pm1(residual(W, B, alpha, z))", "sign_pm1(-residual(W, B, alpha, z))"),
    "expansion_refits_offset": (
        "            alpha, _ = lsq(W, B, z)\n", "            alpha, z = lsq(W, B)\n"),
    "per_precision_variant_keeps_offset": (
        "            alpha, z = lsq(W, B)\n", "            alpha, _ = lsq(W, B)\n"),
    "code_update_farthest": ("idx = np.argmin(err, axis=2)", "idx = np.argmax(err, axis=2)"),
    "code_ties_to_last": (
        "idx = np.argmin(err, axis=2)",
        "idx = err.shape[2] - 1 - np.argmin(err[:, :, ::-1], axis=2)"),
    "candidate_bit_order_reversed": (
        "np.where((c >> np.arange(p)[None, :]) & 1, 1.0, -1.0)",
        "np.where((c >> np.arange(p)[::-1][None, :]) & 1, 1.0, -1.0)"),
    "greedy_scale_over_n_minus_1": (
        "        a = t / n\n", "        a = t / (n - 1)\n"),
    "greedy_from_raw_weights": ("    r = W - z[:, None]\n", "    r = W.copy()\n"),
    "one_round_short": ("    for _ in range(rounds):", "    for _ in range(rounds - 1):"),
    "no_final_refit": (
        "    alpha, z = lsq(W, B)\n    out_alpha", "    out_alpha"),
    "offset_not_refit": (
        "        alpha, z = lsq(W, B)\n        record(\"lsq\"",
        "        alpha, _ = lsq(W, B, z)\n        record(\"lsq\""),
    "dependent_columns_min_norm": (
        "    sol = np.stack([solve_normal_equations(gram[q], rhs[q]) for q in range(P)])",
        "    sol = np.stack([np.linalg.lstsq(gram[q], rhs[q], rcond=None)[0] for q in range(P)])"),
    "adjugate_transposed_cofactor": (
        "[r[:i] + r[i + 1:] for k, r in enumerate(M) if k != j]",
        "[r[:j] + r[j + 1:] for k, r in enumerate(M) if k != i]"),
    "adjugate_sign_pattern": ("(-1) ** (i + j) * det_int", "(-1) ** i * det_int"),
    "cramer_drops_last_term": (
        "        for b in range(1, len(kept)):", "        for b in range(1, len(kept) - 1):"),
    "greedy_ignores_earlier_planes": (
        "            t = t - aj * np.sum(b * bj, axis=1)", "            t = t - 0.0 * aj"),
    "fixed_offset_rhs_sign": (
        "np.einsum(\"qin,qn->qi\", B, W) - z[:, None] * B.sum(axis=2)",
        "np.einsum(\"qin,qn->qi\", B, W) + z[:, None] * B.sum(axis=2)"),
    "offset_column_last": (
        "A = np.concatenate([np.ones((P, 1, n)), B], axis=1)",
        "A = np.concatenate([B, np.ones((P, 1, n))], axis=1)"),
    "packing_msb_first": (
        "words << np.arange(32, dtype=np.uint64)",
        "words << np.arange(31, -1, -1, dtype=np.uint64)"),
    "packing_groups_transposed": (
        "bits = (B > 0).reshape(N, G, p_H, group).transpose(2, 0, 1, 3).reshape(p_H, N, K)",
        "bits = (B > 0).reshape(G, N, p_H, group).transpose(2, 1, 0, 3).reshape(p_H, N, K)"),
    "dependence_test_skips_last_column": (
        "    for j in range(len(G)):", "    for j in range(len(G) - 1):"),
}


def _run_pins(path):
    env = dict(os.environ, BCQ_QUANTIZER_ORACLE=path)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x",
                        "-p", "no:cacheprovider", PINS],
                       cwd=ROOT, env=env, capture_output=True, text=True,
                       timeout=300)
    return r.returncode


@pytest.fixture(scope="module")
def source():
    with open(SRC, encoding="utf-8") as f:
        return f.read()


def _write(d, text):
    path = os.path.join(d, "quantizer_copy.py")
    with open(path, "w", encoding="utf-8") as f:
        f.write(text)
    return path


def test_unmodified_copy_passes(source):
    with tempfile.TemporaryDirectory() as d:
        assert _run_pins(_write(d, source)) == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(source, name):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, f"mutation site for {name} not unique"
    with tempfile.TemporaryDirectory() as d:
        assert _run_pins(_write(d, source.replace(old, new))) != 0

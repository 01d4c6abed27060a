"""Plants plausible mistakes in copies of the oracle and requires the pins to catch each one.

Every mutant is a textual edit of ``oracle/attn_oracle.c`` compiled into a
temporary library (CPU only).  The pins of ``tests/oracle_pins.py`` must fail on
every mutant, which shows they constrain every term of the oracle's formula.
"""
import os
import subprocess

import pytest

import oracle
from tests import oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

MUTANTS = {
    "scale_dropped": ("s[j] = J->scale * dot;", "s[j] = dot;"),
    "exp_sign_flipped": ("double w = exp(s[j] - m);", "double w = exp(m - s[j]);"),
    "exp_base_two": ("double w = exp(s[j] - m);", "double w = exp2(s[j] - m);"),
    "not_normalised": ("out_row[c] = acc[c] / l;", "out_row[c] = acc[c];"),
    "lse_without_max": ("*lse_out = m + log(l);", "*lse_out = log(l);"),
    "lse_log2": ("*lse_out = m + log(l);", "*lse_out = m + log2(l);"),
    "value_head_zero": ("int64_t vbase = ((beg + j) * J->heads + h)", "int64_t vbase = ((beg + j) * J->heads + 0)"),
    "value_of_query_row": ("int64_t vbase = ((beg + j) * J->heads + h)", "int64_t vbase = ((r) * J->heads + h)"),
    "scores_transposed": ("widen(J->q, J->kind, qbase + c) * widen(J->k, J->kind, kbase + c)",
                          "widen(J->q, J->kind, kbase + c) * widen(J->k, J->kind, qbase + c)"),
    "no_block_mask": [("int64_t beg = J->cu[seg], end = J->cu[seg + 1];", "int64_t beg = 0, end = J->total;"),
                      ("(size_t)(J->max_len > 0 ? J->max_len : 1)", "(size_t)(J->total > 0 ? J->total : 1)")],
    "boundary_off_by_one": ("if ((int64_t)cu[mid] <= token) lo = mid;", "if ((int64_t)cu[mid] < token) lo = mid;"),
    "last_key_skipped": ("    for (int64_t j = 0; j < n; ++j) {\n        double w", "    for (int64_t j = 0; j + 1 < n; ++j) {\n        double w"),
    "max_excludes_first_key": ("if (s[j] > m) m = s[j];", "if (j > 0 && s[j] > m) m = s[j];"),
}


def _compile(name, tmp_path):
    src = open(SRC).read()
    edits = MUTANTS[name] if isinstance(MUTANTS[name], list) else [MUTANTS[name]]
    for old, new in edits:
        assert src.count(old) == 1, f"mutation site of {name} not found exactly once"
        src = src.replace(old, new)
    path = tmp_path / f"mut_{name}.c"
    path.write_text(src)
    lib = tmp_path / f"libmut_{name}.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-pthread", "-o", str(lib), str(path), "-lm"],
                   check=True)
    return oracle.bind(str(lib))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    lib = _compile(name, tmp_path)
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"


def test_unmutated_copy_passes(tmp_path):
    path = tmp_path / "copy.c"
    path.write_text(open(SRC).read())
    lib = tmp_path / "libcopy.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-pthread", "-o", str(lib), str(path), "-lm"],
                   check=True)
    for check in pins.ALL_CHECKS:
        check(oracle.bind(str(lib)))

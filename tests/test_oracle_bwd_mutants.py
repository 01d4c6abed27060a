"""Plants plausible mistakes in copies of the gradient oracle and requires the pins to catch each one.

Every mutant is a textual edit of ``oracle/attn_bwd_oracle.c``, compiled with
the unmodified forward oracle into a temporary library (CPU only).
"""
import os
import subprocess

import pytest

import oracle
from tests import oracle_bwd_pins as pins

HERE = os.path.dirname(oracle.__file__)
SRC_FWD = os.path.join(HERE, "attn_oracle.c")
SRC_BWD = os.path.join(HERE, "attn_bwd_oracle.c")

# name -> list of (old, new, expected occurrences)
MUTANTS = {
    "dq_scale_dropped": [("J->dq[IDX(r, h, c, J->d)] += J->scale * ds *", "J->dq[IDX(r, h, c, J->d)] += ds *", 1),
                         ("out[c] += J->scale * ds *", "out[c] += ds *", 1)],
    "dk_scale_dropped": [("J->dk[IDX(beg + j, h, c, J->d)] += J->scale * ds *", "J->dk[IDX(beg + j, h, c, J->d)] += ds *", 1)],
    "delta_dropped": [("double ds = p[j] * (dp[j] - D);", "double ds = p[j] * dp[j];", 2)],
    "delta_sign": [("double ds = p[j] * (dp[j] - D);", "double ds = p[j] * (dp[j] + D);", 2)],
    "weights_not_normalised": [("        p[j] /= l;\n", "", 1)],
    "exp_sign_flipped": [("p[j] = exp(p[j] - m);", "p[j] = exp(m - p[j]);", 1)],
    "score_scale_dropped": [("p[j] = J->scale * dot;", "p[j] = dot;", 1)],
    "dk_from_k": [("J->dk[IDX(beg + j, h, c, J->d)] += J->scale * ds * bwd_widen(J->q, J->kind, IDX(r, h, c, J->d));",
                   "J->dk[IDX(beg + j, h, c, J->d)] += J->scale * ds * bwd_widen(J->k, J->kind, IDX(r, h, c, J->d));", 1)],
    "dq_from_q": [("J->dq[IDX(r, h, c, J->d)] += J->scale * ds * bwd_widen(J->k, J->kind, IDX(beg + j, h, c, J->d));",
                   "J->dq[IDX(r, h, c, J->d)] += J->scale * ds * bwd_widen(J->q, J->kind, IDX(beg + j, h, c, J->d));", 1),
                  ("out[c] += J->scale * ds * bwd_widen(J->k, J->kind, IDX(beg + j, h, c, J->d));",
                   "out[c] += J->scale * ds * bwd_widen(J->q, J->kind, IDX(beg + j, h, c, J->d));", 1)],
    "dv_uses_ds": [("J->dvo[IDX(beg + j, h, c, J->dv)] += p[j] *", "J->dvo[IDX(beg + j, h, c, J->dv)] += (p[j] * (dp[j] - D)) *", 1)],
    "dp_transposed": [("bwd_widen(J->dout, J->kind, IDX(r, h, c, J->dv)) * bwd_widen(J->v, J->kind, IDX(beg + j, h, c, J->dv))",
                       "bwd_widen(J->dout, J->kind, IDX(beg + j, h, c, J->dv)) * bwd_widen(J->v, J->kind, IDX(r, h, c, J->dv))", 1)],
    "no_block_mask": [("int64_t beg = J->cu[seg], end = J->cu[seg + 1], n = end - beg;\n    for (int64_t j = 0; j < n; ++j) {\n        for",
                       "int64_t beg = J->cu[seg], end = J->cu[seg + 1], n = end - beg;\n    int64_t kb = 0, ke = J->total;\n    for (int64_t j = 0; j < n; ++j) {\n        for", 1),
                      ("double D = row_softmax_and_dp(J, r, h, beg, end, p, dp);\n        for (int32_t c = 0; c < J->d; ++c) J->dq",
                       "double D = row_softmax_and_dp(J, r, h, kb, ke, p, dp);\n        for (int32_t c = 0; c < J->d; ++c) J->dq", 1),
                      ("(size_t)(J->max_len > 0 ? J->max_len : 1)", "(size_t)(J->total > 0 ? J->total : 1)", 1),
                      ("        for (int64_t j = 0; j < n; ++j) {\n            double ds = p[j] * (dp[j] - D);\n            for (int32_t c = 0; c < J->d; ++c) {",
                       "        for (int64_t j = beg - kb; j < end - kb; ++j) {\n            double ds = p[j] * (dp[j] - D);\n            for (int32_t c = 0; c < J->d; ++c) {", 1),
                      ("J->dk[IDX(beg + j, h, c, J->d)] += J->scale", "J->dk[IDX(kb + j, h, c, J->d)] += J->scale", 1),
                      ("J->dq[IDX(r, h, c, J->d)] += J->scale * ds * bwd_widen(J->k, J->kind, IDX(beg + j",
                       "J->dq[IDX(r, h, c, J->d)] += J->scale * ds * bwd_widen(J->k, J->kind, IDX(kb + j", 1),
                      ("J->dvo[IDX(beg + j, h, c, J->dv)] += p[j]", "J->dvo[IDX(kb + j, h, c, J->dv)] += p[j]", 1)],
    "last_query_skipped": [("    for (int64_t i = 0; i < n; ++i) {\n        int64_t r = beg + i;",
                            "    for (int64_t i = 0; i + 1 < n; ++i) {\n        int64_t r = beg + i;", 1)],
}


def _compile(src_bwd_text, tmp_path, name):
    path = tmp_path / f"{name}.c"
    path.write_text(src_bwd_text)
    lib = tmp_path / f"lib{name}.so"
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-pthread", "-o", str(lib), SRC_FWD, str(path),
                    "-lm"], check=True)
    return oracle.bind(str(lib))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    src = open(SRC_BWD).read()
    for old, new, count in MUTANTS[name]:
        assert src.count(old) == count, f"mutation site of {name} found {src.count(old)} times, not {count}"
        src = src.replace(old, new)
    lib = _compile(src, tmp_path, f"mut_{name}")
    caught = []
    for check in pins.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, ValueError, FloatingPointError, IndexError):
            caught.append(check.__name__)
    assert caught, f"no pin catches the planted mistake {name}"


def test_unmutated_copy_passes(tmp_path):
    lib = _compile(open(SRC_BWD).read(), tmp_path, "copy")
    for check in pins.ALL_CHECKS:
        check(lib)

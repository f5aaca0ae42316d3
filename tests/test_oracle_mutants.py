"""Plant plausible mistakes in copies of the oracle; each must fail a pin.

Each mutant is the committed ``oracle/qknorm_oracle.c`` with one textual
replacement, compiled by gcc into a temporary directory and driven through
the same ctypes front end.  The committed source is never modified.  A
mutant that passes every pin would show a hole in the pins, so the test
fails then.
"""
import os

import pytest

import oracle
from tests import pins

MUTANTS = {
    "eps_outside_sqrt": ("const double denom = sqrt(m + eps);",
                         "const double denom = sqrt(m) + eps;"),
    "sum_not_mean": ("const double m = s / (double)L;", "const double m = s;"),
    "eps_added_to_sum": ("const double m = s / (double)L;",
                         "const double m = (s + eps) / (double)L - eps;"),
    "no_sqrt": ("const double denom = sqrt(m + eps);", "const double denom = (m + eps);"),
    "gamma_dropped": ("for (int64_t j = 0; j < L; ++j) y[j] = x[j] * g[j] / denom;",
                      "for (int64_t j = 0; j < L; ++j) y[j] = x[j] / denom;"),
    "abs_not_square": ("for (int64_t j = 0; j < L; ++j) s += x[j] * x[j];",
                       "for (int64_t j = 0; j < L; ++j) s += fabs(x[j]);"),
    "sign_lost": ("for (int64_t j = 0; j < L; ++j) y[j] = x[j] * g[j] / denom;",
                  "for (int64_t j = 0; j < L; ++j) y[j] = fabs(x[j]) * g[j] / denom;"),
    "k_heads_use_gamma_q": ("const double *g = (h < Hq) ? gamma_q : gamma_k;",
                            "const double *g = gamma_q;"),
    "head_index_off_by_one": ("const double *g = (h < Hq) ? gamma_q : gamma_k;",
                              "const double *g = (h <= Hq) ? gamma_q : gamma_k;"),
    "gamma_index_shifted": ("for (int64_t j = 0; j < L; ++j) y[j] = x[j] * g[j] / denom;",
                            "for (int64_t j = 0; j < L; ++j) y[j] = x[j] * g[L - 1 - j] / denom;"),
    "layerwise_k_uses_gamma_q": (
        "if (Lk > 0) rmsnorm_row(x + off + Lq, y + off + Lq, gamma_k, Lk, eps);",
        "if (Lk > 0) rmsnorm_row(x + off + Lq, y + off + Lq, gamma_q, Lk, eps);"),
    "layerwise_k_reads_wrong_columns": (
        "if (Lk > 0) rmsnorm_row(x + off + Lq, y + off + Lq, gamma_k, Lk, eps);",
        "if (Lk > 0) rmsnorm_row(x + off + Lk, y + off + Lq, gamma_k, Lk, eps);"),
    "row_stride_ignored": ("const int64_t off = t * row_stride + (int64_t)h * D;",
                           "const int64_t off = t * (int64_t)(Hq + Hk) * D + (int64_t)h * D;"),
    "v_not_copied": ("memcpy(y, x, (size_t)(T * row_stride) * sizeof(double));",
                     "memset(y, 0, (size_t)(T * row_stride) * sizeof(double));"),
    "shard_divides_by_shard_length": ("const double denom = sqrt(S / (double)L + eps);",
                                      "const double denom = sqrt(S / (double)Ls + eps);"),
    "shard_dropped": ("for (int r = 0; r < nshards; ++r) {", "for (int r = 1; r < nshards; ++r) {"),
    "shard_last_only": ("S += Sr;", "S = Sr;"),
}


@pytest.fixture(scope="module")
def source():
    with open(oracle.SOURCE) as f:
        return f.read()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, source, tmp_path):
    old, new = MUTANTS[name]
    assert source.count(old) >= 1, "mutation site vanished: %r" % old
    src = tmp_path / "mutant.c"
    src.write_text(source.replace(old, new, 1))
    lib = oracle.compile_source(str(src), str(tmp_path / ("lib_%s.so" % name)))
    o = oracle.Oracle(lib)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, "mutant %s passed every pin" % name
    assert os.path.exists(lib)

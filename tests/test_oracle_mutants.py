"""Plants plausible mistakes in a copy of the oracle (on the CPU) and checks
that the pins catch every one of them: a pin set that a dropped term, a wrong
sign or index, or a transposed operand slips through would not pin anything."""
import os
import shutil

import pytest

import oracle
import oracle_pins as pins

MUTANTS = {
    "softmax_sign": ("s[j] = exp(s[j] - mx);", "s[j] = exp(mx - s[j]);"),
    "softmax_not_normalised": ("s[j] /= sum;", "s[j] /= 1.0;"),
    "logit_scale_added": ("s[j] = acc;", "s[j] = acc / sqrt((double)d_in);"),
    "value_column_reversed": ("(off + j) * d_emb + e)", "(off + j) * d_emb + (d_emb - 1 - e))"),
    "w_up_transposed": ("elem(W_up, dtype, u * d_emb + e)", "elem(W_up, dtype, e * d_up + u)"),
    "variance_unbiased": ("var /= (double)d_up;", "var /= (double)(d_up - 1);"),
    "mean_not_subtracted": ("((z[u] - mu) * rstd)", "(z[u] * rstd)"),
    "gamma_beta_swapped": ("elem(ln_gamma, dtype, u) * ((z[u] - mu) * rstd) + elem(ln_beta, dtype, u)",
                           "elem(ln_beta, dtype, u) * ((z[u] - mu) * rstd) + elem(ln_gamma, dtype, u)"),
    "residual_dropped": ("for (int64_t i = 0; i < d_in; ++i)\n        acc += elem(W_mix",
                         "for (int64_t i = 0; i < 0; ++i)\n        acc += elem(W_mix"),
    "w_mix_halves_swapped": ("acc += elem(W_mix, dtype, o * ld + u) * h[u];",
                             "acc += elem(W_mix, dtype, o * ld + d_in + u) * h[u];"),
    "previous_token_rows_included": ("int64_t off = offsets[t];", "int64_t off = offsets[t > 0 ? t - 1 : t];"),
    "sort_not_stable": ("for (int64_t n = 0; n < n_tokens; ++n) {\n    int64_t pos",
                        "for (int64_t n = n_tokens - 1; n >= 0; --n) {\n    int64_t pos"),
    "seg_rows_off_by_one": ("seg_rows[g + 1] = (int32_t)rows;", "seg_rows[g + 1] = (int32_t)rows + 1;"),
}


def _caught(lib_path):
    for pin in pins.ALL_PINS:
        try:
            pin(lib_path=lib_path)
        except (AssertionError, oracle.OracleError):
            return pin.__name__
    return None


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "l3_oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = str(tmp_path / "libl3_oracle_mutant.so")
    oracle.compile_library(str(mutated), lib)
    assert _caught(lib) is not None, f"mutant {name} passes every pin"


def test_unmutated_oracle_passes_all_pins():
    assert _caught(oracle.LIBRARY) is None

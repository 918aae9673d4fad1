"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the
pins catch every one: each mutant must fail at least one pin.

The mutants are textual edits of oracle/attn_ref.c compiled into a temporary
library; the real oracle source is never modified."""
import os

import pytest

import oracle
from oracle import build as obuild
from oracle_pins import ALL_PINS

# (name, original text, replacement) -- each a mistake one could plausibly make.
MUTANTS = [
    ("scale_dropped", "srow[j] = scale * dot;", "srow[j] = dot;"),
    ("score_sign", "srow[j] = scale * dot;", "srow[j] = -scale * dot;"),
    ("mask_wrong_side", "for (long j = i + 1; j < Sk; ++j)",
     "for (long j = 0; j < i && j < Sk; ++j)"),
    ("mask_hides_diagonal", "for (long j = i + 1; j < Sk; ++j)", "for (long j = i; j < Sk; ++j)"),
    ("mask_one_late", "for (long j = i + 1; j < Sk; ++j)", "for (long j = i + 2; j < Sk; ++j)"),
    # bottom-right alignment (key j visible to query i when j <= i + Sk - Sq); the
    # edit that threads Sq into the row routine is in _bottom_right_source
    ("mask_bottom_right", "for (long j = i + 1; j < Sk; ++j)", None),
    ("no_max_subtraction", "srow[j] = exp(srow[j] - m);", "srow[j] = exp(srow[j]);"),
    ("lse_without_max", "*lse_i = m + log(l);", "*lse_i = log(l);"),
    ("lse_log2", "*lse_i = m + log(l);", "*lse_i = m + log2(l);"),
    ("value_row_off_by_one", "const double *v_j = vh + j * D;",
     "const double *v_j = vh + (j == 0 ? 0 : j - 1) * D;"),
    ("key_row_wrong", "dot += q_i[d] * kh[j * D + d];",
     "dot += q_i[d] * kh[((j + 1) % Sk) * D + d];"),
    ("feature_reversed", "dot += q_i[d] * kh[j * D + d];",
     "dot += q_i[d] * kh[j * D + (D - 1 - d)];"),
    ("output_row_shifted", "smat + i * Sk, o + (bh * Sq + i) * D,",
     "smat + i * Sk, o + (bh * Sq + (i + 1) % Sq) * D,"),
    ("normaliser_ignored", "srow[j] = srow[j] / l;", "srow[j] = srow[j] / (double)Sk;"),
]


@pytest.fixture(scope="module")
def original_source():
    with open(obuild.SRC) as f:
        return f.read()


def _build_mutant(tmp_path, src, name):
    path = tmp_path / f"mutant_{name}.c"
    path.write_text(src)
    out = tmp_path / f"libmutant_{name}.so"
    obuild.compile_oracle(str(path), str(out))
    return oracle.load(str(out))


def _bottom_right_source(src):
    # the row routine does not see Sq: pass it through a file-scope variable
    src = src.replace("static int attend_one_row(", "static long g_sq;\nstatic int attend_one_row(")
    src = src.replace("if (causal) {\n        for (long j = i + 1; j < Sk; ++j)",
                      "if (causal) {\n        long Sq = g_sq;\n        for (long j = (i + 1 + Sk - Sq > 0 ? i + 1 + Sk - Sq : 0); j < Sk; ++j)")
    src = src.replace("const long heads = B * H;", "const long heads = B * H;\n    g_sq = Sq;")
    src = src.replace("int status = ORACLE_OK;\n#pragma omp parallel\n    {\n        double *srow",
                      "int status = ORACLE_OK;\n    g_sq = Sq;\n#pragma omp parallel\n    {\n        double *srow")
    return src


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, original_source, name, old, new):
    assert old in original_source, f"mutation anchor for {name} not found in the oracle"
    if new is None:
        src = _bottom_right_source(original_source)
        assert src != original_source
    else:
        src = original_source.replace(old, new)
    lib = _build_mutant(tmp_path, src, name)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant {name}"


def test_original_passes_all_pins(oracle_lib):
    for pin in ALL_PINS:
        pin(oracle_lib)

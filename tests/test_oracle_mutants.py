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
MASK_LOOP = "for (long j = (i + 1 + off > 0 ? i + 1 + off : 0); j < Sk; ++j)"
OFFSET = "const long off = (mask == ORACLE_CAUSAL_BOTTOM_RIGHT) ? Sk - Sq : 0;"

# (name, original text, replacement) -- each a mistake one could plausibly make.
MUTANTS = [
    ("scale_dropped", "srow[j] = scale * dot;", "srow[j] = dot;"),
    ("score_sign", "srow[j] = scale * dot;", "srow[j] = -scale * dot;"),
    ("mask_wrong_side", MASK_LOOP, "for (long j = 0; j < i + off && j < Sk; ++j)"),
    ("mask_hides_diagonal", MASK_LOOP,
     "for (long j = (i + off > 0 ? i + off : 0); j < Sk; ++j)"),
    ("mask_one_late", MASK_LOOP,
     "for (long j = (i + 2 + off > 0 ? i + 2 + off : 0); j < Sk; ++j)"),
    # bottom-right alignment applied to the top-left mode
    ("mask_bottom_right", OFFSET, "const long off = Sk - Sq;"),
    ("bottom_right_offset_sign", OFFSET,
     "const long off = (mask == ORACLE_CAUSAL_BOTTOM_RIGHT) ? Sq - Sk : 0;"),
    ("bottom_right_ignored", OFFSET, "const long off = 0;"),
    ("empty_row_lse", "*lse_i = -INFINITY;\n        return ORACLE_OK;",
     "*lse_i = 0.0;\n        return ORACLE_OK;"),
    ("gqa_heads_modulo", "return b * Hkv + h / (H / Hkv);", "return b * Hkv + h % Hkv;"),
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


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, original_source, name, old, new):
    assert original_source.count(old) == 1, f"mutation anchor for {name} not found once"
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

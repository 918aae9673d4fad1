"""The fp64 row-softmax oracle against its pins, and planted mistakes in a copy of
its source (compiled on the CPU) that the pins must catch."""
import pytest

import oracle
from oracle import build as obuild
from softmax_pins import ALL_SOFTMAX_PINS

MUTANTS = [
    ("no_max_subtraction", "y[j] = exp(x[j] - m);", "y[j] = exp(x[j]);"),
    ("max_of_first_only", "if (x[j] > m)\n            m = x[j];", "if (j == 0)\n            m = x[j];"),
    ("normaliser_is_n", "y[j] = y[j] / l;", "y[j] = y[j] / (double)n;"),
    ("sum_skips_last", "for (long j = 0; j < n; ++j) {\n        y[j] = exp(x[j] - m);\n        l += y[j];",
     "for (long j = 0; j < n; ++j) {\n        y[j] = exp(x[j] - m);\n        if (j + 1 < n) l += y[j];"),
    ("input_shifted", "y[j] = exp(x[j] - m);", "y[j] = exp(x[(j + 1) % n] - m);"),
    ("row_stride_wrong", "softmax_one_row(x + r * n, y + r * n, n);",
     "softmax_one_row(x + r * n, y + ((r + 1) % rows) * n, n);"),
]


@pytest.fixture(scope="module")
def softmax_lib():
    return oracle.load_softmax()


@pytest.mark.parametrize("pin", ALL_SOFTMAX_PINS, ids=[p.__name__ for p in ALL_SOFTMAX_PINS])
def test_softmax_oracle_pin(pin, softmax_lib):
    pin(softmax_lib)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_softmax_pins_catch_mutant(tmp_path, name, old, new):
    with open(obuild.SOFTMAX_SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found once"
    path = tmp_path / f"softmax_mutant_{name}.c"
    path.write_text(src.replace(old, new))
    out = tmp_path / f"libsoftmax_mutant_{name}.so"
    obuild.compile_oracle(str(path), str(out))
    lib = oracle.load_softmax(str(out))
    caught = []
    for pin in ALL_SOFTMAX_PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant {name}"

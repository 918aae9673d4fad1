"""The fp64 GEMM + bias + activation oracle against its pins, and planted mistakes in
a copy of its source (compiled on the CPU) that the pins must catch."""
import pytest

import oracle
from oracle import build as obuild
from gemm_pins import ALL_GEMM_PINS

MUTANTS = [
    ("weight_not_transposed", "z += a[m * K + k] * w[n * K + k];",
     "z += a[m * K + k] * w[(k * N + n) % (N * K)];"),
    ("bias_on_rows", "z += bias[n];", "z += bias[m % N];"),
    ("bias_after_activation", "c[m * N + n] = activate(z, act);",
     "c[m * N + n] = activate(z - (bias ? bias[n] : 0.0), act) + (bias ? bias[n] : 0.0);"),
    ("gelu_tanh_form", "return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));",
     "return 0.5 * z * (1.0 + tanh(sqrt(2.0 / 3.141592653589793) * (z + 0.044715 * z * z * z)));"),
    ("gelu_sqrt2_missing", "return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));",
     "return 0.5 * z * (1.0 + erf(z / 2.0));"),
    ("gelu_half_missing", "return 0.5 * z * (1.0 + erf(z / sqrt(2.0)));",
     "return z * (1.0 + erf(z / sqrt(2.0)));"),
    ("relu_leaky", "return z > 0.0 ? z : 0.0;", "return z > 0.0 ? z : 0.01 * z;"),
    ("k_loop_short", "for (long k = 0; k < K; ++k)", "for (long k = 0; k + 1 < K; ++k)"),
]


@pytest.fixture(scope="module")
def gemm_lib():
    return oracle.load_gemm()


@pytest.mark.parametrize("pin", ALL_GEMM_PINS, ids=[p.__name__ for p in ALL_GEMM_PINS])
def test_gemm_oracle_pin(pin, gemm_lib):
    pin(gemm_lib)


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_gemm_pins_catch_mutant(tmp_path, name, old, new):
    with open(obuild.GEMM_SRC) as f:
        src = f.read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found once"
    path = tmp_path / f"gemm_mutant_{name}.c"
    path.write_text(src.replace(old, new))
    out = tmp_path / f"libgemm_mutant_{name}.so"
    obuild.compile_oracle(str(path), str(out))
    lib = oracle.load_gemm(str(out))
    caught = []
    for pin in ALL_GEMM_PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError, FloatingPointError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant {name}"

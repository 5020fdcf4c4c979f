"""The oracle's pins have teeth: each plausible mistake below, planted in a
copy of the oracle's C source and compiled on the CPU, makes at least one pin
of tests/test_oracle_pins.py fail."""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "dfk_oracle.c")

MUTANTS = [
    ("SiLU sign flipped", "a / (1.0 + exp(-a))", "a / (1.0 + exp(a))"),
    ("SiLU on the up branch", "double hv = dfk_oracle_silu(a) * u;",
     "double hv = dfk_oracle_silu(u) * a;"),
    ("eps dropped", "sqrt(ss / (double)D + eps);\n    for (int k = 0; k < D; ++k) {\n      double v",
     "sqrt(ss / (double)D);\n    for (int k = 0; k < D; ++k) {\n      double v"),
    ("mean over D - 1",
     "sqrt(ss / (double)D + eps);\n    for (int k = 0; k < D; ++k) {\n      double v",
     "sqrt(ss / (double)(D - 1) + eps);\n    for (int k = 0; k < D; ++k) {\n      double v"),
    ("rescale without eps", "sqrt(ss / (double)D + eps);\n    for (int k = 0; k < D; ++k) out[",
     "sqrt(ss / (double)D + 1.0);\n    for (int k = 0; k < D; ++k) out["),
    ("gamma not applied", "double o = v * r * g;", "double o = v * r;"),
    ("column-major read as row-major",
     "case ORC_LAYOUT_COL: return dfk_oracle_bf16_to_double(wg[(size_t)k * F + j]);",
     "case ORC_LAYOUT_COL: return dfk_oracle_bf16_to_double(wg[(size_t)j * D + k]);"),
    ("interleaved gate and up swapped",
     "default:             return dfk_oracle_bf16_to_double(wg[(size_t)(2 * j) * D + k]);",
     "default:             return dfk_oracle_bf16_to_double(wg[(size_t)(2 * j + 1) * D + k]);"),
    ("down projection operand transposed",
     "dfk_oracle_bf16_to_double(wd[(size_t)r * F + j])",
     "dfk_oracle_bf16_to_double(wd[(size_t)j * D + r])"),
    ("first reduction term dropped",
     "for (int k = 0; k < D; ++k) {\n        a += xr[k] * w_gate(",
     "for (int k = 1; k < D; ++k) {\n        a += xr[k] * w_gate("),
    ("E4M3 exponent bias 8", "else v = ldexp(1.0 + (double)m / 8.0, e - 7);",
     "else v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    ("E4M3 subnormal scale", "if (e == 0) v = ldexp((double)m, -9);",
     "if (e == 0) v = ldexp((double)m, -10);"),
    ("FP8 row scale ignored",
     "return (double)sc[j] * dfk_oracle_e4m3_to_double(q[(size_t)j * D + k]);",
     "return dfk_oracle_e4m3_to_double(q[(size_t)j * D + k]);"),
    ("ties rounded away from zero",
     "(rem == 0.5 && fmod(fl, 2.0) != 0.0)", "(rem == 0.5)"),
]

PIN_CALLS = []
for name in dir(pins):
    fn = getattr(pins, name)
    if name.startswith("test_") and callable(fn):
        if name in ("test_gate_up_hand_example", "test_gate_up_hand_example_with_rmsnorm"):
            for layout in (0, 1, 2):
                PIN_CALLS.append((name, fn, {"oracle_mod": None, "layout": layout}))
        else:
            PIN_CALLS.append((name, fn, {"oracle_mod": None}))


def failing_pins():
    failed = []
    for name, fn, kw in PIN_CALLS:
        try:
            fn(**kw)
        except Exception:  # an assertion or a rejected argument: the pin caught it
            failed.append(name)
    return failed


def test_pins_pass_on_the_real_oracle():
    oracle._load()
    assert failing_pins() == []


@pytest.mark.parametrize("what,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, what, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation target not unique: %s" % what
    mutant = tmp_path / "mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                    "-shared", "-o", str(lib), str(mutant), "-lm"], check=True)
    with oracle._swapped(str(lib)):
        failed = failing_pins()
    assert failed, "no pin fails when the oracle has: %s" % what

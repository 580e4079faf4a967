"""The oracle's pins catch plausible mistakes.

Each mutant is a copy of the oracle's C source with one deliberate bug patched
in (a dropped term, a wrong sign, a shifted index, a skipped cast, an extra
rounding, a wrong row or column, ties rounded away from zero).  The oracle
itself carries no hook for this: the test rewrites one line of a copy, checks
that the line was there exactly once, compiles the copy and runs the pin suite
against it, which must fail on every mutant.
"""
import os
import subprocess
import sys

import pytest

from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))

# name -> (text in the oracle's source, its replacement)
MUTANTS = {
    "add term dropped": ("const double v = add ? load_elem(out, out_dt, oi) + acc : acc;",
                         "const double v = acc;"),
    "product subtracted": ("acc += xhat[k] * wv;", "acc -= xhat[k] * wv;"),
    "weight row index shifted": ("a * w_as + n * w_ns + k * w_ks", "a * w_as + ((n + 1) % N) * w_ns + k * w_ks"),
    "x not cast to the weight dtype": ("xhat[k] = round_to(load_elem(x, x_dt, r * x_rs + k * x_cs), w_dt);",
                                       "xhat[k] = load_elem(x, x_dt, r * x_rs + k * x_cs);"),
    "product rounded to the weight dtype before the sum": ("acc += xhat[k] * wv;",
                                                           "acc += round_to(xhat[k] * wv, w_dt);"),
    "row index off by one": ("const int64_t r = s + m;", "const int64_t r = s + m + 1;"),
    "slice offset ignored": ("const int64_t oi = r * H + slice_offset + n;", "const int64_t oi = r * H + n;"),
    "ties rounded away from zero": ("(rem == 0.5 && fmod(r, 2.0) != 0.0)", "(rem == 0.5)"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    text, repl = MUTANTS[name]
    src = open(oracle_build.SRC).read()
    assert src.count(text) == 1, f"mutant '{name}': the line to patch is not in the oracle exactly once"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(text, repl))
    lib = oracle_build.build(force=True, out=str(tmp_path / "mutant.so"), src=str(mutant_src))
    env = dict(os.environ, SGMV_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant '{name}' passed every pin"

"""The oracle's pins catch plausible mistakes.

Each mutant is the oracle compiled with one deliberate bug (a dropped term, a
wrong sign, a shifted index, a skipped cast, an extra rounding, a wrong row or
column, ties rounded away from zero).  The pin suite must fail on every one.
"""
import os
import subprocess
import sys

import pytest

from oracle import build as oracle_build

HERE = os.path.dirname(os.path.abspath(__file__))
MUTANTS = {
    1: "add term dropped",
    2: "product subtracted",
    3: "weight row index shifted",
    4: "x not cast to the weight dtype",
    5: "product rounded to the weight dtype before the sum",
    6: "row index off by one",
    7: "slice offset ignored",
    8: "ties rounded away from zero",
}


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_mutant(mutant, tmp_path):
    lib = oracle_build.build(force=True, out=str(tmp_path / f"mutant{mutant}.so"),
                             defines=[f"ORC_MUTANT={mutant}"])
    env = dict(os.environ, SGMV_ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x", "-p", "no:cacheprovider",
                        os.path.join(HERE, "test_oracle_pins.py")],
                       env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {mutant} ({MUTANTS[mutant]}) passed every pin"

"""Compile the CPU oracle (test infrastructure only) into oracle/_liboracle.so.

Usage: python -m oracle.build   (also run by __graft_entry__.build()).
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "sgmv_oracle.c")
LIB = os.path.join(HERE, "_liboracle.so")


def build(force: bool = False, out: str = LIB, src: str = SRC) -> str:
    """Compile the oracle.  `src` other than the oracle's own file is for the
    mutation test only (a patched copy with one deliberate bug)."""
    if not force and src == SRC and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    # -ffp-contract=off: the oracle's products and sums are separate fp64
    # operations, each rounded, exactly as written in the source.
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC",
           "-std=c11", "-Wall", "-o", out + ".tmp", src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force=True))

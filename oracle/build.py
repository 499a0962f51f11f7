"""Compile the C oracle (``bitnet_ref.c``) into ``liboracle_ref.so`` with gcc.

Plain C99, -O2, no fast-math and no FMA contraction, so every fp32 operation
is the single IEEE operation written in the source.  OpenMP only splits the
contraction over output features (each dot product stays sequential).
"""

from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bitnet_ref.c")
LIB = os.path.join(HERE, "liboracle_ref.so")


def build(force: bool = False, verbose: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-fopenmp", SRC, "-o", LIB + ".tmp", "-lm"]
    if verbose:
        print(" ".join(cmd), file=sys.stderr)
    subprocess.run(cmd, check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB



def build_variant(src_text: str, out_path: str) -> str:
    """Compile an edited copy of the oracle source (used by the tests that
    plant mistakes in the oracle to show that its pins catch them)."""
    src = out_path + ".c"
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
                    "-shared", "-w", "-fopenmp", src, "-o", out_path, "-lm"], check=True)
    return out_path


if __name__ == "__main__":
    print(build(force=True, verbose=True))

"""Compile the fp64 CPU oracle (attn_oracle.c) into a shared library.

Test infrastructure only: the oracle is built alongside the CUDA library so the
tests, the smoke check and the bench's CPU-baseline leg can load it; nothing on
the product path links or loads it.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attn_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


def build(out: str = LIB, mutant: int = 0, force: bool = False) -> str:
    """Build the oracle (or, with ``mutant`` > 0, a variant with one planted mistake)."""
    if (not force and mutant == 0 and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SRC)):
        return out
    cmd = ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fopenmp", "-Wall",
           "-Wno-unknown-pragmas", SRC, "-o", out, "-lm"]
    if mutant:
        cmd.insert(1, f"-DORACLE_MUTANT={int(mutant)}")
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

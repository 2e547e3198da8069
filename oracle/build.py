"""Compile the fp64 CPU oracle (plain C, gcc) into oracle/libpa_oracle.so.

Test infrastructure: the product library never links or loads this.
`extra_defines` builds deliberately broken variants (PAO_MUTANT_*) for the tests that check
that the oracle's pins catch plausible mistakes; those go to a caller-chosen path.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "pa_oracle.c")
LIB = os.path.join(HERE, "libpa_oracle.so")


def build(out_path: str = LIB, extra_defines=(), force: bool = False) -> str:
    if (not force and not extra_defines and os.path.exists(out_path)
            and os.path.getmtime(out_path) >= os.path.getmtime(SRC)):
        return out_path
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
           "-ffp-contract=off", "-Wall", "-Wextra", "-Wno-unused-parameter"]
    cmd += [f"-D{d}" for d in extra_defines]
    tmp = out_path + f".tmp{os.getpid()}"
    cmd += [SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out_path)
    return out_path


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

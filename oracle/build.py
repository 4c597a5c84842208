"""Compiles the C oracle (segpaged_oracle.c) into oracle/liboracle.so -- test infrastructure.

Plain gcc, fp64, OpenMP over query rows, ``-ffp-contract=off`` so no multiply-add is fused.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))


def build_oracle(force: bool = False) -> str:
    src = os.path.join(HERE, "segpaged_oracle.c")
    out = os.path.join(HERE, "liboracle.so")
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared", "-std=c11",
                           "-o", tmp, src, "-lm"])
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build_oracle(force=True))

"""Build the oracle's shared library (plain C, fp64) in place.  Test infrastructure only."""
from __future__ import annotations

import os
import subprocess

_DIR = os.path.dirname(os.path.abspath(__file__))


def build() -> str:
    out = os.path.join(_DIR, "liboracle.so")
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-o", out,
           os.path.join(_DIR, "oracle.c"), "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    build()

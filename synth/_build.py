"""Build the host (gcc) and device (nvcc, sm_100a) libraries of the input generator in place."""
from __future__ import annotations

import os
import subprocess

_DIR = os.path.dirname(os.path.abspath(__file__))


def build_host() -> str:
    out = os.path.join(_DIR, "libsynth.so")
    cmd = ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-math-errno", "-fPIC", "-shared",
           "-o", out, os.path.join(_DIR, "synth_host.c"), "-lpthread", "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build_device() -> str:
    out = os.path.join(_DIR, "libsynth_cuda.so")
    cmd = ["nvcc", "-O3", "-std=c++17", "--fmad=false", "-gencode", "arch=compute_100a,code=sm_100a",
           "-lineinfo", "-Xcompiler", "-fPIC", "-shared", "-o", out, os.path.join(_DIR, "synth_dev.cu")]
    subprocess.run(cmd, check=True)
    return out


def build() -> None:
    build_host()
    build_device()


if __name__ == "__main__":
    build()

"""Compile libcsa.so (every .cu under csrc/) for sm_100a, in place."""
from __future__ import annotations

import os
import subprocess
from concurrent.futures import ThreadPoolExecutor

_DIR = os.path.dirname(os.path.abspath(__file__))
_CSRC = os.path.join(_DIR, "csrc")
_OBJ = os.path.join(_DIR, "_build")
LIB = os.path.join(_DIR, "libcsa.so")

NVCC_FLAGS = ["-std=c++17", "-O3", "-gencode", "arch=compute_100a,code=sm_100a", "-lineinfo",
              "-Xcompiler", "-fPIC", "-Xptxas", "-v", "--expt-relaxed-constexpr"]


def sources():
    return sorted(f for f in os.listdir(_CSRC) if f.endswith(".cu"))


def _compile(src: str) -> tuple[str, str]:
    obj = os.path.join(_OBJ, src[:-3] + ".o")
    cmd = ["nvcc", *NVCC_FLAGS, "-c", os.path.join(_CSRC, src), "-o", obj]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError(f"nvcc failed for {src}:\n{r.stdout}\n{r.stderr}")
    return obj, r.stderr


def build(verbose: bool = False) -> str:
    os.makedirs(_OBJ, exist_ok=True)
    with ThreadPoolExecutor(8) as ex:
        res = list(ex.map(_compile, sources()))
    if verbose:
        for _, log in res:
            print(log)
    cmd = ["nvcc", "-shared", "-gencode", "arch=compute_100a,code=sm_100a", "-o", LIB, *[o for o, _ in res],
           "-lcudart"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    build(verbose=True)

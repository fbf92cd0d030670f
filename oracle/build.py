"""Builds the oracle's shared library (oracle/liboracle.so) from oracle.cpp.

Test infrastructure only.  Plain g++, C++17, OpenMP; -ffp-contract=fast lets
each multiply-add step round once; no -ffast-math, so no sum is reordered.
x86-64-v3 (AVX2 + FMA) is the instruction-set floor of the hosts this runs on.
"""
from __future__ import annotations

import os
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")
FLAGS = ["-O3", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-march=x86-64-v3", "-ffp-contract=fast", "-Wall"]


def compile_source(src_text: str | None, out: str, src_path: str = SRC) -> str:
    """Compile oracle source (the file, or `src_text` in its place) into `out`."""
    if src_text is None:
        cmd = ["g++", *FLAGS, src_path, "-o", out]
        r = subprocess.run(cmd, capture_output=True, text=True)
    else:
        with tempfile.NamedTemporaryFile("w", suffix=".cpp", delete=False) as f:
            f.write(src_text)
            tmp = f.name
        try:
            r = subprocess.run(["g++", *FLAGS, tmp, "-o", out], capture_output=True, text=True)
        finally:
            os.unlink(tmp)
    if r.returncode != 0:
        raise RuntimeError(f"oracle build failed:\n{r.stdout}\n{r.stderr}")
    return out


def stale() -> bool:
    return not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if force or stale():
        tmp = LIB + f".tmp{os.getpid()}"
        compile_source(None, tmp)
        os.replace(tmp, LIB)  # atomic: concurrent importers never see a half-written library
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

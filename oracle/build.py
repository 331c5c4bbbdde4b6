"""Build the C++ oracle (``oracle/step.cc``) into ``oracle/liboracle.so``.

TEST INFRASTRUCTURE, like the rest of ``oracle``.  Plain g++, fp64, no BLAS:
``-O2`` and ``-ffp-contract=off`` (no multiply-add fusion, so every sum is the
plain one on any host).  Rebuilds only when the source is newer than the
library.  ``python -m oracle.build`` builds it by hand.
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "step.cc")
LIB = os.path.join(HERE, "liboracle.so")
FLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-pthread", "-ffp-contract=off",
         "-Wall", "-Wextra"]


def compiler() -> str:
    for cand in [os.environ.get("CXX"), shutil.which("g++"), shutil.which("c++")]:
        if cand:
            return cand
    raise RuntimeError("no C++ compiler found for the oracle")


def compile_source(src: str, out: str) -> None:
    """Compile one oracle source file into a shared library at ``out``."""
    tmp = out + f".tmp{os.getpid()}"
    r = subprocess.run([compiler()] + FLAGS + ["-o", tmp, src], capture_output=True,
                       text=True)
    if r.returncode != 0:
        raise RuntimeError(f"oracle build failed:\n{r.stdout}{r.stderr}")
    os.replace(tmp, out)


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        compile_source(SRC, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

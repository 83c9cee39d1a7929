"""Builds the C++ oracle (test infrastructure) into oracle/libcslc_oracle.so.

    python -m oracle.build_oracle

g++ -O2 -fopenmp, C++17; rebuilt when the source is newer than the library.
The first compiler that accepts -fopenmp is used; if none does, the oracle is
built without OpenMP and runs on one thread (orc_threads() reports it).
"""

from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "cslc_oracle.cpp")
LIB = os.path.join(HERE, "libcslc_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cands = [os.environ.get("CXX"), "x86_64-linux-gnu-g++-13", "x86_64-linux-gnu-g++", "g++", "c++"]
    cands = [c for c in cands if c and shutil.which(c)]
    errors = []
    for omp in (["-fopenmp"], []):
        for cxx in cands:
            cmd = [cxx, "-O2", "-std=c++17", *omp, "-fPIC", "-shared", SRC, "-o", LIB + ".tmp"]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode == 0:
                os.replace(LIB + ".tmp", LIB)
                return LIB
            errors.append(f"{' '.join(cmd)}: {r.stderr.strip()[:300]}")
    raise RuntimeError("oracle build failed:\n" + "\n".join(errors))


if __name__ == "__main__":
    print(build(force=True))

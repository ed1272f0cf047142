"""Build the fp64 C++ oracle (``oracle/liboracle.so``) with g++ and OpenMP.

Test infrastructure: the library is loaded only by ``oracle/moba_oracle_c.py``
(tests, ``__graft_entry__.smoke()`` and the CPU legs of ``bench.py``).
``python -m oracle.build_oracle`` rebuilds it when the source is newer.  The
first C++ compiler that builds it with OpenMP is used ($CXX, then the system
g++); without any, it is built single-threaded.
"""
from __future__ import annotations

import os
import shutil
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moba_oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")

# Plain IEEE double arithmetic: no fast-math, no contraction into FMAs.
FLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-ffp-contract=off"]


def _compilers():
    seen = []
    for c in (os.environ.get("CXX"), "/usr/bin/g++", shutil.which("g++")):
        if c and os.path.exists(c) and c not in seen:
            seen.append(c)
    return seen


def build() -> str:
    if os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    errors = []
    for omp in (["-fopenmp"], []):
        for cxx in _compilers():
            cmd = [cxx, *FLAGS, *omp, SRC, "-o", LIB]
            r = subprocess.run(cmd, capture_output=True, text=True)
            if r.returncode == 0:
                return LIB
            errors.append("%s\n%s" % (" ".join(cmd), r.stderr))
    raise RuntimeError("oracle build failed:\n" + "\n".join(errors))


if __name__ == "__main__":
    print(build())

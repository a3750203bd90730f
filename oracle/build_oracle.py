"""Compile the C++ oracle (``moe_oracle.cpp``) into ``oracle/libmoe_oracle.so`` with g++.

Test infrastructure: run by ``__graft_entry__.build()`` (as a script: compiling
the checker, not using it) and on first use by ``moe_oracle.py``.

    python oracle/build_oracle.py [--force]
"""

from __future__ import annotations

import os
import shutil
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "moe_oracle.cpp")
LIB = os.path.join(HERE, "libmoe_oracle.so")
CXX_FLAGS = ["-O2", "-std=c++17", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-Wall"]


def _compilers():
    seen = []
    for c in (shutil.which("g++"), os.environ.get("CXX"), "/usr/bin/g++"):
        if c and c not in seen and os.path.exists(c):
            seen.append(c)
    return seen


def build(force: bool = False) -> str:
    """Compile the oracle (only when the source is newer than the library).

    OpenMP parallelises independent rows only; a compiler without it builds
    the same oracle single-threaded."""
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    tmp = LIB + f".{os.getpid()}.tmp"
    log = []
    for flags in (CXX_FLAGS, [f for f in CXX_FLAGS if f != "-fopenmp"] + ["-Wno-unknown-pragmas"]):
        for cxx in _compilers():
            cmd = [cxx, *flags, SRC, "-o", tmp]
            res = subprocess.run(cmd, capture_output=True, text=True)
            if res.returncode == 0:
                os.replace(tmp, LIB)
                return LIB
            log.append(" ".join(cmd) + "\n" + res.stdout + res.stderr)
    raise RuntimeError("oracle build failed:\n" + "\n".join(log))


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

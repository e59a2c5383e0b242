"""Build the CPU oracle shared library (test infrastructure only).

``build(defines=())`` compiles ``tgemm_oracle.c`` with gcc into ``liboracle.so`` beside
this file, or, when ``defines`` names planted mistakes (``ORACLE_PLANT_*``, used only by
the mutation tests), into a separately named library so the real one is untouched.
"""
from __future__ import annotations

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "tgemm_oracle.c")
HDR = os.path.join(HERE, "tgemm_oracle.h")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
          "-Wall", "-Wextra"]


def lib_path(defines=()) -> str:
    if not defines:
        return os.path.join(HERE, "liboracle.so")
    tag = hashlib.sha1(" ".join(sorted(defines)).encode()).hexdigest()[:10]
    return os.path.join(HERE, "_mutants", f"liboracle_{tag}.so")


def _stale(out: str) -> bool:
    if not os.path.exists(out):
        return True
    t = os.path.getmtime(out)
    return any(os.path.getmtime(p) > t for p in (SRC, HDR, __file__))


def build(defines=(), force: bool = False) -> str:
    out = lib_path(defines)
    if not force and not _stale(out):
        return out
    os.makedirs(os.path.dirname(out), exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", *CFLAGS, *[f"-D{d}" for d in defines], "-o", tmp, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(tuple(sys.argv[1:]), force=True))

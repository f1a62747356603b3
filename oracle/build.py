"""Compiles the C++ CPU oracle (llm_int8.cpp) into liborc_llm_int8.so.

TEST INFRASTRUCTURE ONLY: the oracle is loaded by the tests, the smoke check
and the benchmark's CPU legs, never by the product library.

The flags keep every floating-point operation an IEEE binary32/binary64
operation rounded to nearest even, in source order: no -ffast-math, and
-ffp-contract=off so that no multiply and add are fused.

    python -m oracle.build [--force]
"""
from __future__ import annotations

import os
import shutil
import subprocess
import sys
import tempfile

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "llm_int8.cpp")
LIB = os.path.join(HERE, "liborc_llm_int8.so")
FLAGS = ["-std=c++17", "-O3", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
         "-pthread", "-Wall", "-Wextra"]


def compiler() -> str:
    p = shutil.which("g++") or shutil.which("c++")
    if not p:
        raise RuntimeError("no C++ compiler (g++) found for the CPU oracle")
    return p


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile `src` into the shared library `out` unless it is newer than `src`."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    fd, tmp = tempfile.mkstemp(suffix=".so", dir=os.path.dirname(out))
    os.close(fd)
    try:
        r = subprocess.run([compiler()] + FLAGS + ["-o", tmp, src], capture_output=True, text=True)
        if r.returncode != 0:
            raise RuntimeError("oracle build failed:\n" + r.stdout + r.stderr)
        os.replace(tmp, out)
    finally:
        if os.path.exists(tmp):
            os.unlink(tmp)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

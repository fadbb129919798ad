"""Build the CPU oracle library (test infrastructure): oracle/liboracle_gdn.so,
and the pin-check variant oracle/liboracle_gdn_pincheck.so (the same source
with -DGDN_ORACLE_PIN_CHECK, which adds the entry point that plants known
mistakes; only the pin-sensitivity test loads it)."""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gdn_oracle.c")
LIB = os.path.join(HERE, "liboracle_gdn.so")
LIB_PINCHECK = os.path.join(HERE, "liboracle_gdn_pincheck.so")


def _build(out: str, defines, force: bool) -> str:
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-Wall", "-Wextra", "-fPIC", "-shared", "-pthread",
           *defines, "-o", out, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def build(force: bool = False) -> str:
    return _build(LIB, [], force)


def build_pincheck(force: bool = False) -> str:
    return _build(LIB_PINCHECK, ["-DGDN_ORACLE_PIN_CHECK"], force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv), build_pincheck(force="--force" in sys.argv))

"""Builds the CPU oracle's shared library (test infrastructure only).

gcc, binary64 with no floating-point contraction so every multiply and add rounds
once, OpenMP across independent outputs.
"""
from __future__ import annotations

import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "scope_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")


FLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]
# AddressSanitizer and UndefinedBehaviorSanitizer instrumentation (any report aborts)
SANITIZE = ["-fsanitize=address,undefined", "-fno-sanitize-recover=all", "-fno-omit-frame-pointer", "-g"]


def build(force: bool = False) -> str:
    # SCOPE_ORACLE_LIB: use an already-built library instead (the sanitizer test's build)
    if os.environ.get("SCOPE_ORACLE_LIB"):
        return os.environ["SCOPE_ORACLE_LIB"]
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    subprocess.run(["gcc", *FLAGS, "-o", LIB + ".tmp", SRC, "-lm"], check=True)
    os.replace(LIB + ".tmp", LIB)
    return LIB


def build_sanitized(out: str) -> str:
    """The oracle with ASan + UBSan, to `out` (the process that loads it must preload the
    sanitizer runtimes, e.g. LD_PRELOAD of gcc's libasan.so and libubsan.so)."""
    subprocess.run(["gcc", *FLAGS, *SANITIZE, "-o", out, SRC, "-lm"], check=True)
    return out


if __name__ == "__main__":
    print(build(force=True))

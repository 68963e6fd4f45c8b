"""Build the fp64 CPU oracle (test infrastructure only) into ``oracle/_build/liborc.so``.

Plain gcc, -O2 (no -ffast-math: the oracle's rounding behaviour is part of what it states),
OpenMP over heads.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "gdn_oracle.c")
OUT_DIR = os.path.join(HERE, "_build")
OUT = os.path.join(OUT_DIR, "liborc.so")


def compile_oracle(src: str = SRC, out: str = OUT) -> str:
    """Compile ``src`` into the shared library ``out`` and return ``out``."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-fno-fast-math",
           "-ffp-contract=off", "-Wall", "-Wextra", "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _stale() -> bool:
    return not os.path.exists(OUT) or os.path.getmtime(OUT) < os.path.getmtime(SRC)


def build(force: bool = False) -> str:
    if force or _stale():
        os.makedirs(OUT_DIR, exist_ok=True)
        import fcntl

        with open(os.path.join(OUT_DIR, ".lock"), "w") as lock:  # one builder at a time
            fcntl.flock(lock, fcntl.LOCK_EX)
            if force or _stale():
                tmp = OUT + f".{os.getpid()}.tmp"
                compile_oracle(SRC, tmp)
                os.replace(tmp, OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

"""Build the fp64 CPU oracle library (test infrastructure only).

    python oracle/build.py            # writes oracle/libbsa_oracle.so

Flags keep IEEE fp64 semantics: no fast-math and no FMA contraction, so the
oracle's arithmetic is exactly the order written in bsa_oracle.c.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bsa_oracle.c")
LIB = os.path.join(HERE, "libbsa_oracle.so")

CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-Wall", "-Wextra"]


def build(src: str = SRC, out: str = LIB, extra: list[str] | None = None, force: bool = False) -> str:
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", *CFLAGS, *(extra or []), src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

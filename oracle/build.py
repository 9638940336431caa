"""Build the fp64 CPU oracle library (test infrastructure only).

    python oracle/build.py            # writes oracle/libbsa_oracle.so
    python oracle/build.py --native   # also the host-tuned copy used for CPU timings

Flags keep IEEE fp64 semantics: no fast-math and no FMA contraction, so the
oracle's arithmetic is exactly the order written in bsa_oracle.c. The copy
built for timing (-O3 -march=native, built on the machine that runs it, under
_build/) keeps those two flags, so it computes bit-identical results; without
-ffast-math the compiler may vectorise independent loops but never reassociates
a floating-point sum.
"""
from __future__ import annotations

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "bsa_oracle.c")
LIB = os.path.join(HERE, "libbsa_oracle.so")

CFLAGS = ["-std=c11", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-Wall", "-Wextra"]
NATIVE_FLAGS = ["-O3", "-march=native"]
NATIVE_DIR = os.path.join(os.path.dirname(HERE), "_build", "oracle_native")


def _host_tag() -> str:
    """Short digest of this host's CPU model and feature flags: a -march=native build is only
    reused on a host that reports the same ones."""
    import hashlib
    import platform
    info = platform.machine()
    try:
        with open("/proc/cpuinfo") as f:
            keep = [l for l in f if l.startswith(("model name", "flags"))]
        info += "".join(sorted(set(keep)))
    except OSError:
        pass
    return hashlib.sha256(info.encode()).hexdigest()[:12]


def build(src: str = SRC, out: str = LIB, extra: list[str] | None = None, force: bool = False) -> str:
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    cmd = ["gcc", *CFLAGS, *(extra or []), src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def build_native(force: bool = False) -> str:
    """The timing copy: -O3 -march=native for this host's cores (later flags override -O2)."""
    os.makedirs(NATIVE_DIR, exist_ok=True)
    out = os.path.join(NATIVE_DIR, f"libbsa_oracle_native_{_host_tag()}.so")
    return build(out=out, extra=NATIVE_FLAGS, force=force)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))
    if "--native" in sys.argv:
        print(build_native(force="--force" in sys.argv))

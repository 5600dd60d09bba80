"""Compile the CPU oracle (test infrastructure) into oracle/libckv_oracle.so.

Plain C, strict IEEE order: -O2 -ffp-contract=off -fno-fast-math, so that gcc
neither fuses a*b+c nor reorders sums (the one fmaf in the cluster score is
written out explicitly).
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ckv_oracle.c")
LIB = os.path.join(HERE, "libckv_oracle.so")
FLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
         "-Wall", "-Wextra"]


def build(force: bool = False, out: str = LIB, defines=(), src: str = SRC) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", *FLAGS, *["-D" + x for x in defines], src, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

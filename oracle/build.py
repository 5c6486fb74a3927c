"""Compile the CPU oracle (ep_oracle.c) into oracle/libep_oracle.so.

The oracle is test infrastructure: it is built here so the tests, the smoke check
and the benchmark's CPU-baseline leg can load it.  Plain gcc, no fast-math, no
floating-point contraction, so every product, sum and quotient is one IEEE binary32
operation as written in the source.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ep_oracle.c")
LIB = os.path.join(HERE, "libep_oracle.so")

CFLAGS = ["-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared", "-Wall"]


def build(src=SRC, out=LIB, extra=(), force=False, quiet=True):
    """Build the oracle library; rebuild only when the source is newer unless forced."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", tmp, "-lm"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("oracle build failed:\n%s\n%s" % (" ".join(cmd), res.stderr))
    os.replace(tmp, out)
    if not quiet:
        print(" ".join(cmd))
    return out


if __name__ == "__main__":
    build(force="--force" in sys.argv, quiet=False)

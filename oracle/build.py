"""Compile the CPU oracle (``ep_oracle.c``) into ``liboracle.so`` beside it.

Test infrastructure: the oracle is only built here, loaded by ``oracle/__init__.py``
and used by the tests, the smoke check and the benchmark's CPU-baseline leg.

``-ffp-contract=off`` and the absence of fast-math keep every binary32 operation
a single IEEE-754 rounding, which the oracle's arithmetic relies on.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ep_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-Wall", "-Wextra", "-Werror"]


def build(src=SRC, out=LIB, force=False, extra_flags=()):
    """Build the shared library if it is missing or older than its source."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(src):
        return out
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", *CFLAGS, *extra_flags, "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

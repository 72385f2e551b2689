"""Compile the plain-C oracle into ``oracle/libqz_oracle.so``.

Test infrastructure only (see the header of ``qz_oracle.c``).  The flags keep
IEEE fp32 semantics: no FMA contraction, no fast-math, SSE arithmetic (the
x86-64 default), so every operation rounds once, to nearest-even.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "qz_oracle.c")
LIB = os.path.join(HERE, "libqz_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
          "-shared", "-fopenmp", "-Wall", "-Wextra"]


def build(force: bool = False, src: str = SRC, out: str = LIB, extra=()) -> str:
    """Build the oracle library if it is missing or older than its source."""
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    cmd = ["gcc", *CFLAGS, *extra, src, "-o", out + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

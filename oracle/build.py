"""Build the fp64 CPU oracle into oracle/liboracle.so (plain gcc, OpenMP).

Test infrastructure: the product never loads this library.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "attn_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")

# -O2 without -ffast-math: the compiler may not reassociate the fp64 sums, so
# every dot product and row sum is accumulated in the order the source states.
CFLAGS = ["-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra"]


def build(src=SRC, out=LIB, extra=None, quiet=True):
    """Compile ``src`` into the shared library ``out``; returns its path."""
    cmd = ["gcc", *CFLAGS, *(extra or []), "-o", out, src, "-lm"]
    res = subprocess.run(cmd, capture_output=True, text=True)
    if res.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + " ".join(cmd) + "\n" + res.stderr)
    if not quiet:
        print(" ".join(cmd))
    return out


def needs_build(out=LIB, src=SRC):
    return (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)


if __name__ == "__main__":
    build(quiet=False)
    sys.exit(0)

"""Compile the float64 oracle into oracle/libtitans_oracle.so (gcc, no CUDA).

Test infrastructure: the oracle checks the CUDA library; it is never part of it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "titans_oracle.c")
LIB = os.path.join(HERE, "libtitans_oracle.so")


def compile_source(src: str, out: str) -> str:
    """gcc `src` into the shared library `out` with the oracle's flags."""
    # -ffp-contract=off: no fused multiply-add, so every float64 operation is
    # rounded exactly as written.
    cmd = ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", out + ".tmp", src, "-lpthread", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(out + ".tmp", out)
    return out


def build(force: bool = False) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    return compile_source(SRC, LIB)


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

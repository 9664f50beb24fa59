"""Compile the CPU oracle (``hkv_oracle.c``) into ``libhkv_oracle.so``.

Test infrastructure: the oracle is used only by the test suite, the package
smoke check and the benchmark's CPU-baseline leg.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hkv_oracle.c")
LIB = os.path.join(HERE, "libhkv_oracle.so")


def build(force: bool = False, src: str = SRC, out: str = LIB, extra=()) -> str:
    """Build the oracle shared library with gcc (OpenMP across units)."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= max(
        os.path.getmtime(src), os.path.getmtime(os.path.join(HERE, "hkv_oracle.h"))
    ):
        return out
    cmd = [
        "gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
        "-I", HERE, *extra, src, "-o", out, "-lm",
    ]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

"""Compile the CPU oracle (``moe_oracle.c``) into ``liboracle.so`` next to this file.

The oracle is test infrastructure: it is compiled with gcc, without fast-math and with
floating-point contraction off, so that every fp32 step is one IEEE round-to-nearest
operation and ``fmaf`` appears only where the source writes it.
"""
import os
import pathlib
import subprocess

HERE = pathlib.Path(__file__).resolve().parent
SRC = HERE / "moe_oracle.c"
LIB = HERE / "liboracle.so"

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
          "-shared", "-Wall", "-Wextra", "-Wno-unused-parameter"]


def build(force: bool = False) -> pathlib.Path:
    """Build ``liboracle.so`` if it is missing or older than its source; return its path."""
    if not force and LIB.exists() and LIB.stat().st_mtime >= SRC.stat().st_mtime:
        return LIB
    tmp = LIB.with_suffix(f".so.tmp{os.getpid()}")
    cmd = ["gcc", *CFLAGS, "-o", str(tmp), str(SRC), "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))

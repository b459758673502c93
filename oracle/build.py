"""Compile the CPU oracle (plain C) into oracle/liboracle_hqq.so.

Test infrastructure: the oracle is the CPU restatement that the CUDA library
is checked against.  Building it is not using it.

Flags: -ffp-contract=off keeps every fp32 product and sum separately rounded,
as the C source is written; no -march so that no FMA instruction is emitted.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hqq_oracle.c")
LIB = os.path.join(HERE, "liboracle_hqq.so")


def build(force: bool = False, out: str = LIB, extra_flags=()) -> str:
    """Build the oracle shared library if it is missing or older than its source."""
    if not force and os.path.exists(out) and os.path.getmtime(out) >= os.path.getmtime(SRC):
        return out
    cmd = [
        "gcc", "-std=gnu11", "-O2", "-fPIC", "-shared", "-fopenmp",
        "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra", "-Wno-unused-parameter",
        *extra_flags, SRC, "-o", out, "-lm",
    ]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

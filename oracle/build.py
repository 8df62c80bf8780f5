"""Compile the CPU oracle (test infrastructure only) into oracle/liborc.so.

The oracle is plain C built with -O2 -ffp-contract=off (no fused multiply-add
contraction, no fast-math), so its fp32 decisions are IEEE round-to-nearest-even
operations in program order.  OpenMP only splits independent rows.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "awq_oracle.c")
# AWQ_ORACLE_LIB: a separately built copy to load instead (the sanitizer
# test builds one with -fsanitize=... and points the pins at it)
LIB = os.environ.get("AWQ_ORACLE_LIB") or os.path.join(HERE, "liborc.so")


def build(force: bool = False) -> str:
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math",
           "-fopenmp", "-fPIC", "-shared", "-o", LIB, SRC, "-lm"]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))

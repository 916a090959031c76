"""Build step for the CPU oracle (test infrastructure only).

Compiles ``hq_oracle.c`` into ``libhq_oracle.so`` beside it with strict IEEE
float semantics (no contraction into FMA, no fast-math, no excess precision)
and OpenMP across rows.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "hq_oracle.c")
LIB = os.path.join(HERE, "libhq_oracle.so")

FLAGS = ["-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
         "-fexcess-precision=standard", "-fopenmp", "-lm"]


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its source."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", *FLAGS[:-2], SRC, "-o", tmp, *FLAGS[-2:]])
        os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

"""Build the fp64 CPU oracle (test infrastructure only) into ``oracle/libttt_oracle.so``.

Plain gcc, -O2, IEEE semantics (no fast-math), OpenMP only to spread whole units over threads.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "ttt_oracle.c")
OUT = os.path.join(HERE, "libttt_oracle.so")


def build(force: bool = False) -> str:
    if not force and os.path.exists(OUT) and os.path.getmtime(OUT) >= os.path.getmtime(SRC):
        return OUT
    cmd = ["gcc", "-O2", "-fno-fast-math", "-ffp-contract=off", "-fopenmp", "-shared", "-fPIC",
           "-std=c11", "-D_DEFAULT_SOURCE", "-Wall", "-Wextra", "-o", OUT + ".tmp", SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(OUT + ".tmp", OUT)
    return OUT


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

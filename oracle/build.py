"""Compile the fp64 CPU oracle (lq_oracle.c) into oracle/liblq_oracle.so.

TEST INFRASTRUCTURE: the oracle is only built, loaded and called by the test
suite, the smoke check and the benchmark's CPU-baseline leg.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "lq_oracle.c")
OUT = os.path.join(HERE, "liblq_oracle.so")


def build(force: bool = False, out: str = OUT, defines=()) -> str:
    """Build the oracle shared library; returns its path.

    `defines` adds -D flags (the mutation tests use it to build deliberately
    wrong copies of the oracle into a temporary directory).
    """
    if (not force and not defines and out == OUT and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(SRC)):
        return out
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wextra"]
    cmd += ["-D" + d for d in defines]
    cmd += [SRC, "-o", out, "-lm"]
    subprocess.run(cmd, check=True)
    return out


if __name__ == "__main__":
    print(build(force=True))

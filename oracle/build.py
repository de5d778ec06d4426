"""Build the CPU oracle shared library (test infrastructure only).

Compiles ``wq_oracle.c`` with gcc into ``liboracle.so`` beside it.  The flags
keep every float operation a single IEEE-754 operation: no contraction into
FMA (-ffp-contract=off) and no fast-math.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "wq_oracle.c")
HDR = os.path.join(HERE, "wq_oracle.h")
LIB = os.path.join(HERE, "liboracle.so")


def build(force: bool = False) -> str:
    """Compile the oracle if the library is missing or older than its sources."""
    if not force and os.path.exists(LIB):
        lib_t = os.path.getmtime(LIB)
        if lib_t >= os.path.getmtime(SRC) and lib_t >= os.path.getmtime(HDR):
            return LIB
    cmd = [
        "gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math",
        "-fPIC", "-shared", "-Wall", "-Wextra", "-o", LIB, SRC, "-lm",
    ]
    subprocess.run(cmd, check=True)
    return LIB


if __name__ == "__main__":
    print(build(force=True))

"""Compile the C oracle into a shared object beside its source.

Test infrastructure only: the product library never loads the result.  The flags forbid
floating-point contraction and reassociation, so every step runs in the order the source states.
"""
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "csa_oracle.c")
LIB = os.path.join(HERE, "_csa_oracle.so")

CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off", "-fno-fast-math",
          "-fno-associative-math", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Build the oracle if its shared object is missing or older than the source; return its path."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    subprocess.run(["gcc", *CFLAGS, "-o", tmp, SRC, "-lm"], check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force=True))

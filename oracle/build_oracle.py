"""Build the C part of the CPU oracle (test infrastructure) with gcc.

The oracle library is scalar C compiled with -O2 and no vectorisation flags; it is
loaded through ctypes by ``oracle.t16``.  Nothing in the product path uses it.
"""
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "t16_oracle.c")
LIB = os.path.join(HERE, "liboracle_t16.so")


def build(force: bool = False) -> str:
    """Compile ``t16_oracle.c`` into ``liboracle_t16.so`` next to it; return its path."""
    if (not force and os.path.exists(LIB)
            and os.path.getmtime(LIB) >= os.path.getmtime(SRC)):
        return LIB
    tmp = LIB + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-Wall", "-Wextra",
           "-o", tmp, SRC]
    subprocess.run(cmd, check=True)
    os.replace(tmp, LIB)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv))

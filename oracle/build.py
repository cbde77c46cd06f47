"""Build the CPU oracle library (oracle/libstem_oracle.so) with gcc.

Test infrastructure: the oracle is only loaded by the tests, the smoke check and
the benchmark's CPU-baseline leg.
"""

import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "stem_oracle.c")
LIB = os.path.join(HERE, "libstem_oracle.so")


def build(force: bool = False, quiet: bool = True) -> str:
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall", "-Wextra",
           "-o", LIB, SRC, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + r.stderr)
    if not quiet and r.stderr:
        sys.stderr.write(r.stderr)
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, quiet=False))

"""Build the CPU oracle library (oracle/libstem_oracle.so) with gcc.

Test infrastructure: the oracle is only loaded by the tests, the smoke check and
the benchmark's CPU-baseline leg.

Flags: -O3 -march=native for the host it runs on, OpenMP over rows, and
-ffp-contract=off so that no multiply-add is fused: every expression rounds
exactly as written (the budget's rho(i)*(i+1) must round as in the library's host
code). No -ffast-math: the floating-point semantics stay IEEE.

Because -march=native ties the binary to the build host's instruction set, the
library is rebuilt whenever it was built on a host with another CPU (a stamp file
beside it records the model and instruction-set flags).
"""

import hashlib
import os
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "stem_oracle.c")
LIB = os.path.join(HERE, "libstem_oracle.so")
STAMP = LIB + ".host"
CFLAGS = ["-O3", "-march=native", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
          "-std=c11", "-Wall", "-Wextra"]


def host_id() -> str:
    """The CPU model and instruction-set flags of this host, hashed."""
    model, flags = "", ""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name") and not model:
                    model = line.split(":", 1)[1].strip()
                elif line.startswith("flags") and not flags:
                    flags = " ".join(sorted(line.split(":", 1)[1].split()))
    except OSError:
        pass
    return hashlib.sha256(f"{model}|{flags}|{' '.join(CFLAGS)}".encode()).hexdigest()[:16]


def _current() -> bool:
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        return False
    try:
        with open(STAMP) as f:
            return f.read().strip() == host_id()
    except OSError:
        return False


def build(force: bool = False, quiet: bool = True) -> str:
    if not force and _current():
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    cmd = ["gcc"] + CFLAGS + ["-o", tmp, SRC, "-lm"]
    r = subprocess.run(cmd, capture_output=True, text=True)
    if r.returncode != 0:
        raise RuntimeError("oracle build failed:\n" + r.stderr)
    if not quiet and r.stderr:
        sys.stderr.write(r.stderr)
    os.replace(tmp, LIB)
    with open(STAMP, "w") as f:
        f.write(host_id() + "\n")
    return LIB


if __name__ == "__main__":
    print(build(force="--force" in sys.argv, quiet=False))

"""Writes tests/golden/budget_sums.txt from the oracle alone.

Each line: workload name, nb, rho_min, tau, k_min, sum_i k(i), max_i k(i), k(nb-1).
Regenerate with `python tests/golden/make_golden.py` from the repository root.
"""

import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from block_sparse_causal_pooling_b200.workloads import WORKLOADS  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "budget_sums.txt")


def main():
    lines = ["# name nb rho_min tau k_min sum_k max_k k_last   (written by make_golden.py from the oracle)"]
    for name, w in WORKLOADS.items():
        k, off = oracle.budget(w.nb, w.rho_min, w.tau, w.k_min)
        lines.append(f"{name} {w.nb} {w.rho_min} {w.tau} {w.k_min} {int(off[-1])} {int(k.max())} {int(k[-1])}")
    with open(OUT, "w") as f:
        f.write("\n".join(lines) + "\n")
    print(open(OUT).read())


if __name__ == "__main__":
    main()

"""Writes the oracle-derived golden files of this folder.

Calls only the oracle package.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402

# (n, C, seed, stream id, role) cases of the seeded k-means initialisation.
INIT_CASES = [(1024, 16, 0xC0FFEE + 1, 0, 0), (1024, 16, 0xC0FFEE + 1, 0, 1),
              (8192, 128, 0xC0FFEE + 2, 3, 0), (512, 64, 7, 12, 1), (300, 300, 1, 2, 0),
              (1, 1, 5, 0, 0), (65, 64, 99, 1, 1)]


def main():
    with open(os.path.join(HERE, "init_indices.txt"), "w") as f:
        f.write("# seeded k-means start rows written by make_golden.py from the oracle\n")
        f.write("# format: n C seed sid role : indices\n")
        for n, C, seed, sid, role in INIT_CASES:
            idx = oracle.init_indices(n, C, seed, sid, role)
            f.write(f"{n} {C} {seed} {sid} {role} : " + " ".join(map(str, idx.tolist())) + "\n")


if __name__ == "__main__":
    main()

"""Writes the stored oracle values under tests/golden/ (calls only oracle/ and
the seeded generators).  Run from the repository root:

    python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle as O  # noqa: E402
import workloads as W  # noqa: E402

ROWS = (0, 1, 48, 96, 97)


def main():
    x = W.three_tone(16000, seed=0)
    L, M = O.log_mel(x, return_energy=True)
    assert L.shape == (98, 128)
    path = os.path.join(HERE, "three_tone_1s_rows.txt")
    with open(path, "w") as f:
        f.write("# oracle log-mel of the seeded 1 s three-tone clip (workloads.three_tone, seed 0)\n")
        f.write("# rows: frame index followed by 128 float64 values (repr)\n")
        for r in ROWS:
            f.write(f"{r} " + " ".join(repr(float(v)) for v in L[r]) + "\n")
    print("wrote", path)


if __name__ == "__main__":
    main()

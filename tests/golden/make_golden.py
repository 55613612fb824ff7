"""Write tests/golden/formula_case_expected.txt with the FP64 oracle.

    python tests/golden/make_golden.py

Calls only oracle/ (and the formula inputs).  Stores heads 0, 5, 17 and 31
of every sequence, 17 significant digits.
"""
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from tests.golden import formula_case as fc  # noqa: E402

HEADS = (0, 5, 17, 31)


def main():
    q, pool = fc.inputs()
    out = oracle.decode(q, pool, fc.BT, fc.LENS, 0, fc.SCALE, nthreads=1)
    path = os.path.join(HERE, "formula_case_expected.txt")
    with open(path, "w") as f:
        f.write("# FP64 oracle output for tests/golden/formula_case.py (written by make_golden.py)\n")
        f.write("# columns: sequence head d value\n")
        for b in range(fc.LENS.size):
            for h in HEADS:
                for d in range(64):
                    f.write("%d %d %d %.17g\n" % (b, h, d, out[b, h, d]))
    print(path)


if __name__ == "__main__":
    main()
